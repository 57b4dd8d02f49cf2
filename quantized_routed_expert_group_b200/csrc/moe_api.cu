// moe_api.cu -- the library's C ABI (include/moe.h): argument validation,
// workspace layout and the launch sequence of one MoE layer forward.
#include <cmath>
#include <cstring>
#include <mutex>
#include <unordered_set>

#include <nvtx3/nvToolsExt.h>

#include "moe_internal.h"

#define MOE_API extern "C" __attribute__((visibility("default")))

namespace moe {

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

Layout make_layout(const moe_config& c, int T) {
    Layout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align256(off + bytes);
        return o;
    };
    const size_t t = (size_t)T, H = (size_t)c.hidden, I = (size_t)c.inter, E = (size_t)c.n_experts,
                 k = (size_t)c.top_k;
    const size_t slots = t * k + t * (size_t)c.n_shared;
    L.err = take(64);
    L.ctrl = take(kFusedCtrlBytes);  // fixed offset: the fused path keeps it across calls
    L.xin = take(t * H * 4);
    L.outbuf = take(t * H * 4);
    L.xq = take(t * H);
    L.xd = take(t * (H / 32) * 4);
    L.logits = take(router_ws_bytes(c, T));
    L.idx = take(t * k * 4);
    L.idx_ep = take(t * k * 4);
    L.w = take(t * k * 4);
    L.counts = take(E * 4);
    L.offsets = take((E + 1) * 4);
    L.perm = take(t * k * 4);
    L.inv_perm = take(t * k * 4);
    L.active = take((E + 2) * 4);
    L.hbuf = take(slots * I * 4);
    L.hq = take(slots * I);
    L.hd = take(slots * (I / 32) * 4);
    L.y = take(slots * H * 4);
    if (tc_path_supported(c, T)) {
        const TcSizes z = tc_sizes(c, T);
        const size_t pr = (size_t)z.prows_cap;
        L.tc_xg = take(pr * H);
        L.tc_xdT = take((H / 32) * pr * 8);
        L.tc_gu = take(2 * pr * I * 4);
        L.tc_hg = take(pr * I);
        L.tc_hdT = take((I / 32) * pr * 8);
        L.tc_xp = take(pr * 5 * H);
        L.tc_hp = take(pr * 5 * I);
        L.tc_pex = take(pr * 8);
        L.tc_peh = take(pr * 8);
        L.tc_xpt = take(t * 5 * H);
        L.tc_pet = take(t * 8);
        L.tc_row_tok = take(pr * 4);
        L.tc_row_slot = take(pr * 4);
        L.tc_units_gu = take((size_t)z.units_gu_cap * kTcUnitBytes);
        L.tc_units_dn = take((size_t)z.units_dn_cap * kTcUnitBytes);
        L.tc_ctrl = take(64);
    } else {
        L.tc_xg = L.tc_xdT = L.tc_gu = L.tc_hg = L.tc_hdT = L.tc_row_tok = L.tc_row_slot = 0;
        L.tc_xp = L.tc_hp = L.tc_pex = L.tc_peh = L.tc_xpt = L.tc_pet = 0;
        L.tc_units_gu = L.tc_units_dn = L.tc_ctrl = 0;
    }
    L.total = off;
    return L;
}

const DeviceInfo& device_info() {
    static DeviceInfo infos[64];
    static bool done[64];
    static std::mutex mu;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    std::lock_guard<std::mutex> lock(mu);
    if (!done[dev]) {
        DeviceInfo d{148, 227 * 1024};
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) d.sm_count = v;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) == cudaSuccess && v > 0)
            d.max_smem_optin = v;
        infos[dev] = d;
        done[dev] = true;
    }
    return infos[dev];
}

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

static int check_config(const moe_config* c) {
    if (!c) return MOE_EINVAL;
    if (c->hidden <= 0 || c->inter <= 0 || c->n_experts <= 0 || c->n_groups <= 0 || c->topk_groups <= 0 ||
        c->top_k <= 0 || c->n_shared < 0)
        return MOE_EINVAL;
    if (c->n_experts % c->n_groups != 0 || c->topk_groups > c->n_groups) return MOE_EINVAL;
    if (c->top_k > c->topk_groups * (c->n_experts / c->n_groups)) return MOE_EINVAL;
    if (!std::isfinite(c->routed_scaling_factor)) return MOE_EINVAL;
    if (!std::isfinite(c->expert_topp) || c->expert_topp < 0.f) return MOE_EINVAL;
    if (c->hidden % 32 || c->inter % 32 || c->hidden > 16384 || c->inter > 16384) return MOE_EUNSUPPORTED;
    if (c->n_experts > 1024 || c->n_groups > 32 || c->n_experts / c->n_groups < 2 || c->top_k > 32 ||
        c->n_shared > 1)
        return MOE_EUNSUPPORTED;
    if (c->wbits != 4 && c->wbits != 8 && c->wbits != 2) return MOE_EUNSUPPORTED;
    return MOE_OK;
}

static int check_experts(const moe_experts* ex) {
    if (!ex) return MOE_EINVAL;
    if (!ex->w_gate || !ex->w_up || !ex->w_down || !ex->s_gate || !ex->s_up || !ex->s_down) return MOE_EINVAL;
    if (!aligned(ex->w_gate, 16) || !aligned(ex->w_up, 16) || !aligned(ex->w_down, 16)) return MOE_EINVAL;
    if (!aligned(ex->s_gate, 4) || !aligned(ex->s_up, 4) || !aligned(ex->s_down, 4)) return MOE_EINVAL;
    return MOE_OK;
}

static int status_of(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ECUDA; }

// NVTX range around the launches of one forward phase, so that a profiler
// can select a phase's kernels (ncu --nvtx --nvtx-include "moe/fused/").
// Without an attached tool the calls return at once.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// Per-thread tracing events (see moe_profile_events).
static thread_local cudaEvent_t g_trace[MOE_PROFILE_MAX_EVENTS];
static thread_local bool g_trace_on = false;

static cudaError_t trace(int i, cudaStream_t s) {
    return g_trace_on ? record_event(g_trace[i], s) : cudaSuccess;
}

static int check_bucket_fits(const moe_config& c, int T) {
    if (T > (1 << 20)) return MOE_EUNSUPPORTED;
    const size_t words = (size_t)c.n_experts * (size_t)((T + 31) / 32);
    if (words > 24576) return MOE_EUNSUPPORTED;
    if (bucket_smem_bytes(c, T) > (size_t)device_info().max_smem_optin) return MOE_EUNSUPPORTED;
    return MOE_OK;
}

// The forward on a device-resident x; used by both public forwards.
// ep_lo, ep_hi: the routed experts this call computes (all: 0, n_experts);
// the picks outside the range are routed as usual but left to another call.
// The fused path's control region of a workspace is initialised on the
// first fused forward this process issues with it (or by moe_workspace_init);
// the process remembers the regions it has initialised.  Initialising again
// is always correct: no call uses the region meanwhile (calls that share a
// workspace are ordered on one stream).
static int ensure_fused_ctrl(int* ctrl, cudaStream_t s, bool force) {
    static std::mutex mu;
    static std::unordered_set<uint64_t> seen;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ECUDA;
    const uint64_t key = ((uint64_t)(uint32_t)dev << 56) ^ (uint64_t)reinterpret_cast<uintptr_t>(ctrl);
    std::lock_guard<std::mutex> lock(mu);
    if (!force && seen.count(key)) return MOE_OK;
    if (launch_fused_ctrl_init(ctrl, s) != cudaSuccess) return MOE_ECUDA;
    if (seen.size() >= 4096) seen.clear();
    seen.insert(key);
    return MOE_OK;
}

static int forward_device(const moe_config& c, const float* x, int T, const float* router_w,
                          const float* router_bias, const moe_experts& routed, const moe_experts* shared,
                          float* out, char* ws, const Layout& L, cudaStream_t s, int ep_lo, int ep_hi) {
    int32_t* err = reinterpret_cast<int32_t*>(ws + L.err);
    int8_t* xq = reinterpret_cast<int8_t*>(ws + L.xq);
    float* xd = reinterpret_cast<float*>(ws + L.xd);
    int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
    float* w = reinterpret_cast<float*>(ws + L.w);
    int32_t* counts = reinterpret_cast<int32_t*>(ws + L.counts);
    int32_t* offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
    int32_t* perm = reinterpret_cast<int32_t*>(ws + L.perm);
    int32_t* inv_perm = reinterpret_cast<int32_t*>(ws + L.inv_perm);
    int32_t* active = reinterpret_cast<int32_t*>(ws + L.active);
    if (small_path_supported(c, T)) {
        const NvtxRange range("moe/fused");
        SmallArgs a;
        a.cfg = &c;
        a.T = T;
        a.x = x;
        a.router_w = router_w;
        a.bias = router_bias;
        a.routed = routed;
        a.shared = shared ? *shared : routed;
        a.xq = xq;
        a.xd = xd;
        a.logits = reinterpret_cast<double*>(ws + L.logits);
        a.idx = idx;
        a.w = w;
        a.counts = counts;
        a.offsets = offsets;
        a.perm = perm;
        a.inv_perm = inv_perm;
        a.active = active;
        a.hbuf = reinterpret_cast<float*>(ws + L.hbuf);
        a.hq = reinterpret_cast<int8_t*>(ws + L.hq);
        a.hd = reinterpret_cast<float*>(ws + L.hd);
        a.y = reinterpret_cast<float*>(ws + L.y);
        a.out = out;
        a.ctrl = reinterpret_cast<int*>(ws + L.ctrl);
        a.err = err;
        a.ep_lo = ep_lo;
        a.ep_hi = ep_hi;
        int st2 = ensure_fused_ctrl(a.ctrl, s, false);
        if (!st2) st2 = status_of(trace(0, s));
        if (!st2) st2 = status_of(launch_small(a, s));
        if (!st2) st2 = status_of(trace(1, s));
        return st2;
    }
    const NvtxRange range("moe/multi_kernel");
    if (trace(0, s) != cudaSuccess) return MOE_ECUDA;
    if (cudaMemsetAsync(err, 0, 64, s) != cudaSuccess) return MOE_ECUDA;  // also the batched path's wide flags
    const bool tc = tc_path_supported(c, T);
    int st = tc ? status_of(launch_tc_quantize(x, T, c.hidden, xq, xd, reinterpret_cast<int8_t*>(ws + L.tc_xpt),
                                               reinterpret_cast<double*>(ws + L.tc_pet), err + 8, s))
                : status_of(launch_quantize_q8_0(x, T, c.hidden, xq, xd, s));
    if (st) return st;
    st = status_of(launch_router(c, x, T, router_w, router_bias, reinterpret_cast<double*>(ws + L.logits), idx, w, s));
    if (!st) st = status_of(trace(1, s));
    if (st) return st;
    const int32_t* bidx = idx;  // the picks this call computes
    if (ep_lo > 0 || ep_hi < c.n_experts) {
        int32_t* idx_ep = reinterpret_cast<int32_t*>(ws + L.idx_ep);
        st = status_of(launch_ep_mask(idx, (int64_t)T * c.top_k, ep_lo, ep_hi, idx_ep, s));
        if (st) return st;
        bidx = idx_ep;
    }
    st = status_of(launch_bucket(c, bidx, T, counts, offsets, perm, inv_perm, active, err, s));
    if (st) return st;
    TcArgs ta{};
    if (tc) {
        ta.xg = reinterpret_cast<int8_t*>(ws + L.tc_xg);
        ta.xdT = reinterpret_cast<double*>(ws + L.tc_xdT);
        ta.gu = reinterpret_cast<float*>(ws + L.tc_gu);
        ta.hg = reinterpret_cast<int8_t*>(ws + L.tc_hg);
        ta.hdT = reinterpret_cast<double*>(ws + L.tc_hdT);
        ta.xp = reinterpret_cast<int8_t*>(ws + L.tc_xp);
        ta.hp = reinterpret_cast<int8_t*>(ws + L.tc_hp);
        ta.pex = reinterpret_cast<double*>(ws + L.tc_pex);
        ta.peh = reinterpret_cast<double*>(ws + L.tc_peh);
        ta.xpt = reinterpret_cast<int8_t*>(ws + L.tc_xpt);
        ta.pet = reinterpret_cast<double*>(ws + L.tc_pet);
        ta.xwide = err + 8;
        ta.hwide = err + 9;
        ta.row_tok = reinterpret_cast<int32_t*>(ws + L.tc_row_tok);
        ta.row_slot = reinterpret_cast<int32_t*>(ws + L.tc_row_slot);
        ta.units_gu = ws + L.tc_units_gu;
        ta.units_dn = ws + L.tc_units_dn;
        ta.ctrl = reinterpret_cast<int32_t*>(ws + L.tc_ctrl);
        ta.sz = tc_sizes(c, T);
    }
    ExpertArgs a;
    a.cfg = &c;
    a.T = T;
    a.xq = xq;
    a.xd = xd;
    a.w = w;
    a.offsets = offsets;
    a.perm = perm;
    a.inv_perm = inv_perm;
    a.active = active;
    a.routed = routed;
    a.shared = shared ? *shared : routed;
    a.hq = reinterpret_cast<int8_t*>(ws + L.hq);
    a.hd = reinterpret_cast<float*>(ws + L.hd);
    a.y = reinterpret_cast<float*>(ws + L.y);
    a.out = out;
    a.err = err;
    if (tc) {
        ta.ex = a;
        st = status_of(launch_tc_prepare(ta, s));
        if (!st) st = status_of(trace(2, s));
        if (st) return st;
        return status_of(launch_tc_experts(ta, s, g_trace_on ? &g_trace[3] : nullptr));
    }
    if (trace(2, s) != cudaSuccess) return MOE_ECUDA;
    return status_of(launch_experts(a, s, g_trace_on ? &g_trace[3] : nullptr));
}

static int check_forward_args(const moe_config* cfg, const void* x, int T, const float* router_w,
                              const float* router_bias, const moe_experts* routed, const moe_experts* shared,
                              const void* out, const void* workspace, size_t ws_bytes, Layout* L) {
    int st = check_config(cfg);
    if (st) return st;
    if (T < 0) return MOE_EINVAL;
    if (T > 0 && (!x || !out)) return MOE_EINVAL;  // empty batches may pass null activations
    if (!router_w || !router_bias || !workspace) return MOE_EINVAL;
    if (!aligned(router_w, 16) || !aligned(router_bias, 4) || !aligned(workspace, 256)) return MOE_EINVAL;
    st = check_experts(routed);
    if (st) return st;
    if (cfg->n_shared) {
        st = check_experts(shared);
        if (st) return st;
    }
    st = check_bucket_fits(*cfg, T);
    if (st) return st;
    *L = make_layout(*cfg, T);
    if (ws_bytes < L->total) return MOE_EWORKSPACE;
    return MOE_OK;
}

}  // namespace moe

using namespace moe;

MOE_API int moe_quantize_act_q8_0(const float* x, int64_t n_rows, int cols, int8_t* q, float* d, void* stream) {
    if (n_rows < 0 || cols <= 0 || cols % 32) return MOE_EINVAL;
    if (n_rows == 0) return MOE_OK;
    if (!x || !q || !d || !aligned(x, 4) || !aligned(d, 4)) return MOE_EINVAL;
    return status_of(launch_quantize_q8_0(x, n_rows, cols, q, d, (cudaStream_t)stream));
}

MOE_API int moe_pack_weights(const float* w, int64_t rows, int cols, int wbits, uint8_t* packed, float* scales,
                             void* stream) {
    if (rows < 0 || cols <= 0 || cols % 32) return MOE_EINVAL;
    if (wbits != 8 && wbits != 4 && wbits != 2) return MOE_EUNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (!w || !packed || !scales || !aligned(w, 16) || !aligned(packed, 16) || !aligned(scales, 4))
        return MOE_EINVAL;
    return status_of(launch_pack_weights(w, rows, cols, wbits, packed, scales, (cudaStream_t)stream));
}

MOE_API int moe_requant_fp8(const uint8_t* w_fp8, const float* block_scales, int64_t rows, int cols, int block,
                            int wbits, uint8_t* packed, float* scales, void* stream) {
    if (rows < 0 || cols <= 0 || cols % 32 || block <= 0 || block % 32) return MOE_EINVAL;
    if (wbits != 8 && wbits != 4 && wbits != 2) return MOE_EUNSUPPORTED;
    if (rows == 0) return MOE_OK;
    if (!w_fp8 || !block_scales || !packed || !scales || !aligned(w_fp8, 4) || !aligned(block_scales, 4) ||
        !aligned(packed, 16) || !aligned(scales, 4))
        return MOE_EINVAL;
    return status_of(
        launch_requant_fp8(w_fp8, block_scales, rows, cols, block, wbits, packed, scales, (cudaStream_t)stream));
}

MOE_API size_t moe_router_workspace_bytes(const moe_config* cfg, int T) {
    if (check_config(cfg) != MOE_OK || T < 0 || T > (1 << 20)) return 0;
    return align256(router_ws_bytes(*cfg, T));
}

MOE_API int moe_router_select(const moe_config* cfg, const float* x, int T, const float* router_w,
                              const float* router_bias, int32_t* idx, float* w, void* workspace, size_t ws_bytes,
                              void* stream) {
    int st = check_config(cfg);
    if (st) return st;
    if (T < 0) return MOE_EINVAL;
    if (T == 0) return MOE_OK;
    if (!x || !router_w || !router_bias || !idx || !w || !workspace) return MOE_EINVAL;
    if (!aligned(x, 16) || !aligned(router_w, 16) || !aligned(workspace, 256)) return MOE_EINVAL;
    if (ws_bytes < moe_router_workspace_bytes(cfg, T)) return MOE_EWORKSPACE;
    return status_of(launch_router(*cfg, x, T, router_w, router_bias, reinterpret_cast<double*>(workspace), idx,
                                   w, (cudaStream_t)stream));
}

MOE_API int moe_bucket_tokens(const moe_config* cfg, const int32_t* idx, int T, int32_t* counts, int32_t* offsets,
                              int32_t* perm, void* stream) {
    int st = check_config(cfg);
    if (st) return st;
    if (T < 0) return MOE_EINVAL;
    if (!counts || !offsets || (T > 0 && (!idx || !perm))) return MOE_EINVAL;
    st = check_bucket_fits(*cfg, T);
    if (st) return st;
    // inv_perm and the active-expert list are internal to the forward: not written here.
    return status_of(launch_bucket(*cfg, idx, T, counts, offsets, perm, nullptr, nullptr, nullptr,
                                   (cudaStream_t)stream));
}

MOE_API size_t moe_workspace_bytes(const moe_config* cfg, int T_max) {
    if (check_config(cfg) != MOE_OK || T_max < 0) return 0;
    if (check_bucket_fits(*cfg, T_max) != MOE_OK) return 0;  // no forward runs that many tokens
    return make_layout(*cfg, T_max).total;
}

MOE_API int moe_workspace_init(const moe_config* cfg, int T_max, void* workspace, size_t ws_bytes, void* stream) {
    int st = check_config(cfg);
    if (st) return st;
    if (T_max < 0 || !workspace) return MOE_EINVAL;
    const Layout L = make_layout(*cfg, T_max);
    if (ws_bytes < L.total) return MOE_EWORKSPACE;
    return ensure_fused_ctrl(reinterpret_cast<int*>(static_cast<char*>(workspace) + L.ctrl), (cudaStream_t)stream,
                             true);
}

MOE_API int moe_layer_forward(const moe_config* cfg, const float* x, int T, const float* router_w,
                              const float* router_bias, const moe_experts* routed, const moe_experts* shared,
                              float* out, void* workspace, size_t ws_bytes, void* stream) {
    Layout L;
    int st = check_forward_args(cfg, x, T, router_w, router_bias, routed, shared, out, workspace, ws_bytes, &L);
    if (st) return st;
    if (T == 0) return MOE_OK;
    if (!aligned(x, 16) || !aligned(out, 4)) return MOE_EINVAL;
    return forward_device(*cfg, x, T, router_w, router_bias, *routed, cfg->n_shared ? shared : nullptr, out,
                          static_cast<char*>(workspace), L, (cudaStream_t)stream, 0, cfg->n_experts);
}

MOE_API int moe_layer_forward_partial(const moe_config* cfg, const float* x, int T, const float* router_w,
                                      const float* router_bias, const moe_experts* routed, const moe_experts* shared,
                                      int expert_lo, int expert_hi, int with_shared, float* out, void* workspace,
                                      size_t ws_bytes, void* stream) {
    int st = check_config(cfg);
    if (st) return st;
    if (expert_lo < 0 || expert_hi < expert_lo || expert_hi > cfg->n_experts) return MOE_EINVAL;
    if (with_shared != 0 && with_shared != 1) return MOE_EINVAL;
    moe_config c = *cfg;  // the shared expert only where this call adds it
    if (!with_shared) c.n_shared = 0;
    // the workspace is the full layer's (it is at least this call's)
    Layout L;
    st = check_forward_args(cfg, x, T, router_w, router_bias, routed, with_shared ? shared : routed, out, workspace,
                            ws_bytes, &L);
    if (st) return st;
    if (T == 0) return MOE_OK;
    if (!aligned(x, 16) || !aligned(out, 4)) return MOE_EINVAL;
    // the full layer's layout (every region is at least this call's), so
    // moe_workspace_view(cfg, T) describes this call's intermediates too
    return forward_device(c, x, T, router_w, router_bias, *routed, c.n_shared ? shared : nullptr, out,
                          static_cast<char*>(workspace), L, (cudaStream_t)stream, expert_lo, expert_hi);
}

MOE_API int moe_layer_forward_host(const moe_config* cfg, const float* x_host, int T, const float* router_w,
                                   const float* router_bias, const moe_experts* routed, const moe_experts* shared,
                                   float* out_host, void* workspace, size_t ws_bytes, void* stream) {
    Layout L;
    int st = check_forward_args(cfg, x_host, T, router_w, router_bias, routed, shared, out_host, workspace,
                                ws_bytes, &L);
    if (st) return st;
    if (T == 0) return MOE_OK;
    cudaStream_t s = (cudaStream_t)stream;
    char* ws = static_cast<char*>(workspace);
    const size_t bytes = (size_t)T * cfg->hidden * sizeof(float);
    float* xdev = reinterpret_cast<float*>(ws + L.xin);
    float* odev = reinterpret_cast<float*>(ws + L.outbuf);
    if (cudaMemcpyAsync(xdev, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return MOE_ECUDA;
    st = forward_device(*cfg, xdev, T, router_w, router_bias, *routed, cfg->n_shared ? shared : nullptr, odev, ws, L,
                        s, 0, cfg->n_experts);
    if (st) return st;
    if (cudaMemcpyAsync(out_host, odev, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ECUDA;
    return status_of(cudaStreamSynchronize(s));
}

// ---------------------------------------------------------------------------
// Allocation-free forward: the scratch is a fixed file-scope device array.
// In host code g_noalloc_scratch names a host-side stand-in, not the device
// array, so its device address is looked up with cudaGetSymbolAddress, once
// per device, with that device current, and passed to the kernels.
// ---------------------------------------------------------------------------
MOE_API int moe_get_device_error(void* workspace, void* stream, int32_t* code);

constexpr size_t kNoallocScratchBytes = (size_t)8 << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

static void* noalloc_scratch_address(int* status) {
    static void* addr[64];
    static bool ready[64];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        *status = MOE_ECUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!ready[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
            *status = MOE_ECUDA;
            return nullptr;
        }
        addr[dev] = p;
        ready[dev] = true;
    }
    *status = MOE_OK;
    return addr[dev];
}

MOE_API int moe_layer_forward_noalloc(const moe_config* cfg, const float* x, int T, const float* router_w,
                                      const float* router_bias, const moe_experts* routed,
                                      const moe_experts* shared, float* out, void* stream) {
    int st = check_config(cfg);
    if (st) return st;
    if (T < 0) return MOE_EINVAL;
    st = check_bucket_fits(*cfg, T);  // also keeps the layout arithmetic below in range
    if (st) return st;
    if (make_layout(*cfg, T).total > kNoallocScratchBytes) return MOE_EWORKSPACE;
    void* scratch = noalloc_scratch_address(&st);
    if (st) return st;
    Layout L;
    st = check_forward_args(cfg, x, T, router_w, router_bias, routed, shared, out, scratch, kNoallocScratchBytes,
                            &L);
    if (st) return st;
    if (T == 0) return MOE_OK;
    if (!aligned(x, 16) || !aligned(out, 4)) return MOE_EINVAL;
    return forward_device(*cfg, x, T, router_w, router_bias, *routed, cfg->n_shared ? shared : nullptr, out,
                          static_cast<char*>(scratch), L, (cudaStream_t)stream, 0, cfg->n_experts);
}

MOE_API int moe_noalloc_device_error(void* stream, int32_t* code) {
    if (!code) return MOE_EINVAL;
    int st = MOE_OK;
    void* scratch = noalloc_scratch_address(&st);
    if (st) return st;
    // the error word is the first word of the layout, whatever the config
    return moe_get_device_error(scratch, stream, code);
}

MOE_API int moe_workspace_view(const moe_config* cfg, int T, void* workspace, size_t ws_bytes,
                               moe_workspace_layout* view) {
    int st = check_config(cfg);
    if (st) return st;
    if (T < 0 || !workspace || !view) return MOE_EINVAL;
    st = check_bucket_fits(*cfg, T);
    if (st) return st;
    const Layout L = make_layout(*cfg, T);
    if (ws_bytes < L.total) return MOE_EWORKSPACE;
    char* ws = static_cast<char*>(workspace);
    view->xq = reinterpret_cast<int8_t*>(ws + L.xq);
    view->xd = reinterpret_cast<float*>(ws + L.xd);
    view->idx = reinterpret_cast<int32_t*>(ws + L.idx);
    view->w = reinterpret_cast<float*>(ws + L.w);
    view->counts = reinterpret_cast<int32_t*>(ws + L.counts);
    view->offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
    view->perm = reinterpret_cast<int32_t*>(ws + L.perm);
    view->hq = reinterpret_cast<int8_t*>(ws + L.hq);
    view->hd = reinterpret_cast<float*>(ws + L.hd);
    view->y = reinterpret_cast<float*>(ws + L.y);
    view->error = reinterpret_cast<int32_t*>(ws + L.err);
    return MOE_OK;
}

MOE_API int moe_block_dots(const uint8_t* packed, int64_t rows, int cols, int wbits, const int8_t* q, int n,
                           int32_t* out, void* stream) {
    if (rows < 0 || n < 0 || cols <= 0 || cols % 32) return MOE_EINVAL;
    if (wbits != 4 && wbits != 8 && wbits != 2) return MOE_EUNSUPPORTED;
    if (rows == 0 || n == 0) return MOE_OK;
    if (!packed || !q || !out || !aligned(packed, 16) || !aligned(q, 16) || !aligned(out, 4)) return MOE_EINVAL;
    return status_of(launch_block_dots(packed, rows, cols, wbits, q, n, out, (cudaStream_t)stream,
                                       MOE_DOTS_MULTI_KERNEL));
}

MOE_API int moe_block_dots_routine(const uint8_t* packed, int64_t rows, int cols, int wbits, const int8_t* q, int n,
                                   int routine, int32_t* out, void* stream) {
    if (routine != MOE_DOTS_MULTI_KERNEL && routine != MOE_DOTS_FUSED && routine != MOE_DOTS_TENSOR)
        return MOE_EUNSUPPORTED;
    if (rows < 0 || n < 0 || cols <= 0 || cols % 32) return MOE_EINVAL;
    if (wbits != 4 && wbits != 8 && wbits != 2) return MOE_EUNSUPPORTED;
    if (routine == MOE_DOTS_TENSOR && (n > 64 || ((int64_t)cols * wbits / 8) % 16 || rows > 0x7FFFFFFF))
        return MOE_EUNSUPPORTED;
    if (rows == 0 || n == 0) return MOE_OK;
    if (!packed || !q || !out || !aligned(packed, 16) || !aligned(q, 16) || !aligned(out, 4)) return MOE_EINVAL;
    if (routine == MOE_DOTS_TENSOR)
        return status_of(launch_tc_block_dots(packed, rows, cols, wbits, q, n, out, (cudaStream_t)stream));
    return status_of(launch_block_dots(packed, rows, cols, wbits, q, n, out, (cudaStream_t)stream, routine));
}

MOE_API int moe_get_device_error(void* workspace, void* stream, int32_t* code) {
    if (!workspace || !code) return MOE_EINVAL;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ECUDA;
    *code = v;
    return v == 0 ? MOE_OK : MOE_EDEVICE;
}

MOE_API int moe_debug_fault_injection(int withhold_entry, int64_t wait_budget_ns) {
    if (withhold_entry < -1 || wait_budget_ns < 0 || wait_budget_ns > (int64_t)10 * 1000 * 1000 * 1000)
        return MOE_EINVAL;
    set_fault_injection(withhold_entry, wait_budget_ns);
    return MOE_OK;
}

MOE_API int moe_debug_down_rows(const moe_config* cfg, int T, int n_entries, int grid, int32_t* starts,
                                int* row_cap) {
    if (check_config(cfg) != MOE_OK || !starts || !row_cap) return MOE_EINVAL;
    const int max_ent = 1 + (cfg->n_experts < T * cfg->top_k ? cfg->n_experts : T * cfg->top_k);
    if (T < 1 || T > 4 || n_entries < 1 || n_entries > max_ent || grid < 1 || grid > 4096) return MOE_EINVAL;
    *row_cap = small_down_rows(*cfg, T, n_entries, grid, starts);
    return MOE_OK;
}

MOE_API int moe_synth_normal(uint64_t seed, uint64_t tid, int64_t offset, int64_t n, float sigma, float* out,
                             void* stream) {
    if (n < 0 || offset < 0) return MOE_EINVAL;
    if (n == 0) return MOE_OK;
    if (!out || !aligned(out, 4)) return MOE_EINVAL;
    return status_of(launch_synth_normal(seed, tid, offset, n, sigma, out, (cudaStream_t)stream));
}

MOE_API int moe_profile_events(void* const* events, int n_events) {
    if (!events) {
        if (n_events != 0) return MOE_EINVAL;
        g_trace_on = false;
        return MOE_OK;
    }
    if (n_events != MOE_PROFILE_MAX_EVENTS) return MOE_EINVAL;
    for (int i = 0; i < MOE_PROFILE_MAX_EVENTS; ++i) {
        if (!events[i]) return MOE_EINVAL;
        g_trace[i] = static_cast<cudaEvent_t>(events[i]);
    }
    g_trace_on = true;
    return MOE_OK;
}

MOE_API int moe_forward_launches(const moe_config* cfg, int T) {
    const int st = check_config(cfg);
    if (st) return st;
    if (T < 0) return MOE_EINVAL;
    if (T == 0) return 0;
    if (small_path_supported(*cfg, T)) return kSmallLaunches;
    if (tc_path_supported(*cfg, T)) return kTcLaunches;
    return kForwardLaunches + (router_splits(*cfg, T) > 0 ? 1 : 0);
}

MOE_API int moe_forward_phases(const moe_config* cfg, int T) {
    const int st = check_config(cfg);
    if (st) return st;
    if (T < 0) return MOE_EINVAL;
    if (T == 0) return 0;
    return small_path_supported(*cfg, T) ? 1 : 5;
}

MOE_API const char* moe_forward_phase_name(const moe_config* cfg, int T, int i) {
    static const char* multi[5] = {"route", "bucket", "gate_up", "down", "combine"};
    const int n = moe_forward_phases(cfg, T);
    if (i < 0 || i >= n) return "";
    return n == 1 ? "fused" : multi[i];
}

MOE_API const char* moe_status_string(int status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_EINVAL: return "MOE_EINVAL: invalid argument";
        case MOE_EUNSUPPORTED: return "MOE_EUNSUPPORTED: unsupported shape or bit width";
        case MOE_EWORKSPACE: return "MOE_EWORKSPACE: workspace too small";
        case MOE_ECUDA: return "MOE_ECUDA: CUDA call failed";
        case MOE_EDEVICE: return "MOE_EDEVICE: a kernel recorded a fault";
        default: return "unknown moe status";
    }
}
