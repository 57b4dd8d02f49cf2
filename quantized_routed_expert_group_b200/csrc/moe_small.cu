// moe_small.cu -- the whole MoE layer forward for small batches (T <= 4:
// decode and speculative verify) as one persistent kernel.
//
// What it computes is the layer of moe_api.cu (router, batch-union bucketing,
// SwiGLU experts on Q8_0 activations, combine; GeekNews "Show HN: 느린 컴퓨터에서
// GLM 5.2 실행하기", §구현된 주요 기능; wpnews.pro "Colibri — รัน GLM-5.2 ...",
// spec and kernel tables, "Batch-Union MoE").  How it is scheduled is B200's:
//
// * At one to four tokens the layer is a stream of ~170-360 MB of expert
//   weights, so the goal is to keep HBM busy from the first cycle to the
//   last.  Each CTA (one per SM) has a producer warp that streams work items
//   with bulk asynchronous copies (cp.async.bulk, the 1-D TMA form) into a
//   ring of 48 KB shared-memory slots, and eight consumer warps doing the
//   integer dots on __dp4a.
// * Items come from one global queue in dependency order: router rows,
//   SELECT, shared-expert gate/up rows, QUANTISE(shared), routed gate/up rows,
//   QUANTISE(routed), shared down rows, routed down rows, COMBINE.  An item
//   only waits on items with smaller queue indices, which running CTAs have
//   already taken, so no wait can deadlock; every wait is bounded and records
//   an error code when it runs out.
// * Nothing on the consumers' path waits for a global round trip: they signal
//   completion with fire-and-forget release reductions; the waiting is done by
//   the producer of the item that depends on them (it polls, then copies the
//   inputs the item needs - h rows, h codes, partial outputs - into its slot).
// * The producer prefetches its next queue index one item ahead and keeps the
//   routing schedule in shared memory, so issuing an item costs no round trip.
// * COMBINE sums the per-expert outputs of a tile of rows in a fixed order in
//   fp64: no float atomics, results are bit-reproducible.
// * A tiny prologue kernel (Q8_0 of x, control-block reset) runs first; the
//   main kernel is launched as its programmatic dependent and prefetches its
//   first, routing-independent item before waiting for it.
#include <cmath>

#include "moe_device.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kSmallThreads = kConsumers + 32;
constexpr int kSlotWeightBytes = 48 * 1024;
constexpr int kMaxSlots = 4;
// Bounds of every wait (legitimate waits last microseconds): mbarrier
// try_wait iterations, and polls of a global word with a short sleep each.
constexpr uint32_t kWaitLimit = 1u << 20;
constexpr uint32_t kSpinLimit = 1u << 21;
// Consumers only ever wait for their producer, whose own waits are bounded
// and end in a DONE marker, so their bound is far larger and never reached
// unless the device misbehaves.
constexpr uint32_t kConsumerWaitLimit = 1u << 24;
// Per-item completion signals: every consumer warp of an item adds one.
constexpr int kWarpSignals = kConsumerWarps;

enum ItemKind : int {
    kItemRouter = 1,
    kItemSelect = 2,
    kItemGateUp = 3,
    kItemQuant = 4,
    kItemDown = 5,
    kItemCombine = 6,
    kItemDone = 7
};

// Control block (int32 words, zeroed by the prologue on every call):
// [queue, router_done, routing, -, gu_done[nent], hq_ready[nent], tile_done[n_dn]]
enum : int { kCQueue = 0, kCRouterDone = 1, kCRouting = 2, kCHeader = 4 };

struct SmallGeom {
    int nent;       // 1 + max routed entries (entry 0 = shared expert)
    int n_router;   // router items (2 experts each)
    int rg;         // gate/up rows per item (per matrix)
    int ks;         // K-splits per gate/up row (warps per row)
    int n_gu;       // gate/up items per expert
    int rd;         // down rows per item (= combine tile)
    int n_dn;       // down items per expert (= output tiles)
    int n_static;   // items per CTA taken before the queue (0 or 1)
    int pos_sel;    // queue index of SELECT
    int n_fixed;    // items before the routing-dependent part
    int nslot;      // ring slots
    int act_bytes;  // per-slot activation area (down items)
    int slot_bytes;
    int ctrl_words;
    int sched_words;  // routing schedule record (after the control words)
    int sched_w_off;  // word offset of the padded weights inside the record
    int tk_pad;       // T*k rounded up to 4
    int smem_bytes;
    int tmax;
};

struct SmallParams {
    int T, H, I, E, G, tg, k, ns, wbits;
    float rsf;
    const float* x;
    const float* router_w;
    const float* bias;
    moe_experts routed;
    moe_experts shared;
    int8_t* xq;
    float* xd;
    double* logits;
    int32_t* idx;
    float* w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* perm;
    int32_t* inv_perm;
    int32_t* active;
    float* hbuf;
    int8_t* hq;
    float* hd;
    float* y;
    float* out;
    int* ctrl;
    int* sched;
    int32_t* err;
    SmallGeom g;
};

struct SlotMeta {
    int kind;
    int entry;   // 0 shared, 1 + a routed
    int expert;  // routed expert id; -1 shared; first expert for router items
    int row0;
    int nrows;
    int n;       // tokens
    int slot0;   // first h / y slot
    int aux;     // down: byte offset of the h scales in the activation area
    int tok[4];
};

// ---------------------------------------------------------------------------
// Geometry
// ---------------------------------------------------------------------------
static int round_up(int v, int a) { return (v + a - 1) / a * a; }
__host__ __device__ __forceinline__ int round_up_dev(int v, int a) { return (v + a - 1) / a * a; }

SmallGeom small_geometry(const moe_config& c, int T, int sm_count) {
    SmallGeom g{};
    const int H = c.hidden, I = c.inter, E = c.n_experts;
    const int rbI = I * c.wbits / 8;
    g.tmax = T <= 1 ? 1 : T <= 2 ? 2 : 4;
    g.nent = 1 + (E < T * c.top_k ? E : T * c.top_k);
    g.n_router = (E + 1) / 2;
    g.ks = c.wbits == 8 ? 2 : 1;
    g.rg = kConsumerWarps / g.ks;
    g.n_gu = I / g.rg;
    int rd = kSlotWeightBytes / rbI;
    rd = rd > 64 ? 64 : rd;
    g.rd = rd / 8 * 8;
    g.n_dn = (H + g.rd - 1) / g.rd;
    const int n_sgu = c.n_shared ? g.n_gu : 0;
    g.n_static = (g.n_router + n_sgu) >= sm_count ? 1 : 0;
    const int S = g.n_static * sm_count;
    g.pos_sel = S > g.n_router ? S : g.n_router;
    g.n_fixed = g.n_router + 1 + (c.n_shared ? n_sgu + 1 : 0);
    g.nslot = g.tmax == 1 ? 4 : 3;
    g.act_bytes = round_up(g.tmax * I + g.tmax * (I / 32) * 4 + 32 + 64 * 4, 128);
    g.slot_bytes = kSlotWeightBytes + g.act_bytes;
    g.ctrl_words = round_up(kCHeader + 2 * g.nent + g.n_dn, 4);
    g.tk_pad = round_up(T * c.top_k, 4);
    g.sched_w_off = round_up(1 + 8 * (g.nent - 1), 4);
    g.sched_words = g.sched_w_off + 2 * g.tk_pad;
    const int nb = H / 32;
    const int xq_bytes = round_up(g.tmax * H, 128);
    const int xd_bytes = round_up(g.tmax * nb * 4, 128);
    const int scratch = 8192;
    g.smem_bytes = g.nslot * g.slot_bytes + xq_bytes + xd_bytes + scratch;
    return g;
}

bool small_path_supported(const moe_config& c, int T) {
    if (T < 1 || T > 4) return false;
    if (c.hidden > 6144 || c.n_experts > 256 || c.n_groups > 32 || c.top_k > 32) return false;
    const int rbI = c.inter * c.wbits / 8;
    if (8 * rbI > kSlotWeightBytes) return false;
    const int tmax = T <= 1 ? 1 : T <= 2 ? 2 : 4;
    if (tmax * c.inter * 4 > kSlotWeightBytes) return false;  // h rows of a QUANTISE item
    return small_geometry(c, T, 148).smem_bytes <= device_info().max_smem_optin;
}

size_t small_ctrl_bytes(const moe_config& c, int T) {
    const SmallGeom g = small_geometry(c, T > 0 ? T : 1, 148);
    return (size_t)(g.ctrl_words + g.sched_words) * 4;
}

// ---------------------------------------------------------------------------
// Prologue: reset the control block and quantise x (launches its dependent
// right away so the main kernel can start prefetching).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_small_prologue(const float* __restrict__ x, int64_t nblk,
                                                        int8_t* __restrict__ xq, float* __restrict__ xd, int* ctrl,
                                                        int ctrl_words, int32_t* err) {
    pdl_launch_dependents();
    const int gtid = blockIdx.x * blockDim.x + threadIdx.x;
    for (int i = gtid; i < ctrl_words; i += gridDim.x * blockDim.x) ctrl[i] = 0;
    if (gtid == 0) *err = 0;
    const int lane = threadIdx.x & 31;
    for (int64_t b = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); b < nblk; b += (int64_t)gridDim.x * 8) {
        int8_t q;
        float d;
        q8_0_warp(x[b * kQBlock + lane], q, d);
        xq[b * kQBlock + lane] = q;
        if (lane == 0) xd[b] = d;
    }
}

// ---------------------------------------------------------------------------
// Shared-memory layout of the main kernel
// ---------------------------------------------------------------------------
struct SmemPtrs {
    uint8_t* slots;
    uint8_t* xq;   // [tmax][2][nb][16]: each 32-code block split in halves
    float* xd;     // [tmax][nb]
    uint64_t* full;
    uint64_t* empty;
    SlotMeta* meta;
    double* rpart;  // [2][4][4]
    float* gpart;   // [4][2][8]
    int* sel_idx;   // [4][32]
    int* cnt;       // [256]
    int* off;       // [260]
    int* flags;     // [16] broadcast words
    int* sched;     // producer's copy of the routing schedule record [1 + 8*128]
};

__device__ __forceinline__ SmemPtrs carve(uint8_t* base, const SmallGeom& g, int H) {
    SmemPtrs s;
    uint8_t* p = base;
    s.slots = p;
    p += g.nslot * g.slot_bytes;
    s.xq = p;
    p += round_up_dev(g.tmax * H, 128);
    s.xd = reinterpret_cast<float*>(p);
    p += round_up_dev(g.tmax * (H / 32) * 4, 128);
    s.full = reinterpret_cast<uint64_t*>(p);
    p += 8 * kMaxSlots;
    s.empty = reinterpret_cast<uint64_t*>(p);
    p += 8 * kMaxSlots;
    s.rpart = reinterpret_cast<double*>(p);
    p += sizeof(double) * 32;
    s.meta = reinterpret_cast<SlotMeta*>(p);
    p += sizeof(SlotMeta) * kMaxSlots;
    s.gpart = reinterpret_cast<float*>(p);
    p += sizeof(float) * 64;
    s.sel_idx = reinterpret_cast<int*>(p);
    p += sizeof(int) * 128;
    s.cnt = reinterpret_cast<int*>(p);
    p += sizeof(int) * 256;
    s.off = reinterpret_cast<int*>(p);
    p += sizeof(int) * 260;
    s.flags = reinterpret_cast<int*>(p);
    p += sizeof(int) * 16;
    s.sched = reinterpret_cast<int*>(p);
    return s;
}

// ---------------------------------------------------------------------------
// Producer: the whole warp runs the loop in lockstep; lane 0 alone touches the
// queue, the barriers and the copy engine, the other lanes help with polls of
// many words and with loading the routing schedule.
// ---------------------------------------------------------------------------
struct Producer {
    const SmallParams& p;
    SmemPtrs& s;
    const int lane;
    uint64_t pol;
    int slot = 0;
    uint32_t pe = 1;  // parity to wait on the empty barriers (fresh ring: all empty)
    bool routed_known = false;
    bool aborted = false;  // a wait ran out: stop issuing, drain and exit
    int U = 0;
    uint64_t hq_ready_lo = 0, hq_ready_hi = 0, hq_ready_top = 0;  // entries 0..63, 64..127, 128
    uint32_t issued_mask = 0, issued_par = 0;  // per slot: a copy was issued / its phase parity

    __forceinline__ __device__ Producer(const SmallParams& p_, SmemPtrs& s_, int lane_) : p(p_), s(s_), lane(lane_) {
        pol = l2_evict_first_policy();
    }

    __forceinline__ __device__ void mark_issued() {
        issued_mask |= 1u << slot;
        issued_par = (issued_par & ~(1u << slot)) | ((pe ^ 1u) << slot);
    }

    __forceinline__ __device__ void advance() {
        if (++slot == p.g.nslot) {
            slot = 0;
            pe ^= 1u;
        }
    }

    __forceinline__ __device__ void fail() {
        if (lane == 0) set_error(p.err, kErrTimeout);
        aborted = true;
    }

    bool need_proxy_fence = false;  // set after acquiring data that the next copies read

    // Poll until *f >= target (lane 0 polls; the result is broadcast).
    __forceinline__ __device__ bool wait_geq(const int* f, int target) {
        int ok = 0;
        need_proxy_fence = true;
        if (lane == 0) {
            for (uint32_t i = 0; i < kSpinLimit; ++i) {
                if (ld_acquire_gpu(f) >= target) {
                    ok = 1;
                    break;
                }
                __nanosleep(64);
            }
        }
        ok = __shfl_sync(kFull, ok, 0);
        __syncwarp();
        if (!ok) fail();
        return ok != 0;
    }

    __forceinline__ __device__ bool entry_ready(int e) const {
        if (e < 64) return (hq_ready_lo >> e) & 1ull;
        if (e < 128) return (hq_ready_hi >> (e - 64)) & 1ull;
        return hq_ready_top != 0;
    }

    // Wait until entry e's h codes are published; every poll reads all
    // entries' flags at once (one round trip for the whole warp).
    __forceinline__ __device__ bool wait_hq(int e) {
        const int* flags = p.ctrl + kCHeader + p.g.nent;
        if (!entry_ready(e)) need_proxy_fence = true;
        for (uint32_t it = 0; it < kSpinLimit && !entry_ready(e); ++it) {
            const bool f0 = lane < p.g.nent && ld_acquire_gpu(flags + lane) >= kWarpSignals;
            const bool f1 = lane + 32 < p.g.nent && ld_acquire_gpu(flags + lane + 32) >= kWarpSignals;
            const bool f2 = lane + 64 < p.g.nent && ld_acquire_gpu(flags + lane + 64) >= kWarpSignals;
            const bool f3 = lane + 96 < p.g.nent && ld_acquire_gpu(flags + lane + 96) >= kWarpSignals;
            const bool f4 = lane == 0 && 128 < p.g.nent && ld_acquire_gpu(flags + 128) >= kWarpSignals;
            hq_ready_lo = (uint64_t)__ballot_sync(kFull, f0) | ((uint64_t)__ballot_sync(kFull, f1) << 32);
            hq_ready_hi = (uint64_t)__ballot_sync(kFull, f2) | ((uint64_t)__ballot_sync(kFull, f3) << 32);
            hq_ready_top = __ballot_sync(kFull, f4);
            if (!entry_ready(e)) __nanosleep(128);
        }
        __syncwarp();
        if (!entry_ready(e)) {
            fail();
            return false;
        }
        return true;
    }

    __forceinline__ __device__ bool know_routing() {
        if (routed_known) return true;
        if (!wait_geq(p.ctrl + kCRouting, 1)) return false;
        const int words = 1 + 8 * (p.g.nent - 1);
        for (int i = lane; i < words; i += 32) s.sched[i] = __ldcg(p.sched + i);
        __syncwarp();
        const int umax = p.g.nent - 1;
        const int u = s.sched[0];
        U = u < 0 ? 0 : (u > umax ? umax : u);
        routed_known = true;
        return true;
    }

    // Tokens of an entry: 0 = shared (every token), 1 + a = routed expert a.
    __forceinline__ __device__ void entry_tokens(SlotMeta& m, int entry) {
        if (entry == 0) {
            m.expert = -1;
            m.slot0 = p.T * p.k;
            m.n = p.T;
            for (int i = 0; i < 4; ++i) m.tok[i] = i < p.T ? i : 0;
            return;
        }
        const int* r = s.sched + 1 + 8 * (entry - 1);
        int e = r[0], n = r[2];
        m.expert = (e < 0 || e >= p.E) ? 0 : e;
        m.slot0 = r[1] < 0 ? 0 : r[1];
        m.n = n < 0 ? 0 : (n > p.g.tmax ? p.g.tmax : n);
        for (int i = 0; i < 4; ++i) {
            const int t = r[3 + i];
            m.tok[i] = (t < 0 || t >= p.T) ? 0 : t;
        }
    }

    // Issue item q (called by the whole warp); returns false once it has
    // issued the DONE marker or aborted.
    __forceinline__ __device__ bool issue(int q) {
        if (aborted) return false;
        const SmallGeom& g = p.g;
        SlotMeta m;
        m.kind = kItemDone;
        m.entry = 0;
        m.expert = -1;
        m.row0 = 0;
        m.nrows = 0;
        m.n = 0;
        m.slot0 = 0;
        m.aux = 0;
        for (int i = 0; i < 4; ++i) m.tok[i] = 0;
        const int64_t rowH = (int64_t)p.H * p.wbits / 8, rowI = (int64_t)p.I * p.wbits / 8;
        const int n_sgu = p.ns ? g.n_gu : 0;
        // at most 3 fixed copies, plus one per output slot for COMBINE
        const void *src0 = nullptr, *src1 = nullptr, *src2 = nullptr, *src3 = nullptr;
        uint32_t by0 = 0, by1 = 0, by2 = 0, by3 = 0;
        uint32_t dof0 = 0, dof1 = 0, dof2 = 0, dof3 = 0;
        int ncopy = 0;
        bool combine_copies = false;
        if (q < g.n_router) {
            m.kind = kItemRouter;
            m.expert = 2 * q;
            m.nrows = (p.E - 2 * q) < 2 ? (p.E - 2 * q) : 2;
            src0 = p.router_w + (int64_t)m.expert * p.H;
            by0 = (uint32_t)(m.nrows * p.H * 4);
            ncopy = 1;
        } else if (q == g.pos_sel) {
            m.kind = kItemSelect;
        } else if (q < g.n_router + n_sgu + 1) {
            const int i = q < g.pos_sel ? q - g.n_router : q - g.n_router - 1;
            m.kind = kItemGateUp;
            m.entry = 0;
            m.row0 = i * g.rg;
            m.nrows = g.rg;
            entry_tokens(m, 0);
            src0 = p.shared.w_gate + (int64_t)m.row0 * rowH;
            src1 = p.shared.w_up + (int64_t)m.row0 * rowH;
            by0 = by1 = (uint32_t)(g.rg * rowH);
            dof1 = by0;
            src2 = p.shared.s_gate + m.row0;
            src3 = p.shared.s_up + m.row0;
            by2 = by3 = (uint32_t)(g.rg * 4);
            dof2 = kSlotWeightBytes;
            dof3 = kSlotWeightBytes + 64;
            ncopy = 4;
        } else {
            int entry = -1;  // QUANTISE entry
            if (p.ns && q == g.n_router + n_sgu + 1) {
                entry = 0;
            } else {
                if (!know_routing()) return finish();
                int r = q - g.n_fixed;
                // gate/up items of entry b, each followed by the QUANTISE of
                // entry b-1 (one entry of lag, so that its inputs are done):
                // G(0) | G(1) Q(0) | G(2) Q(1) | ... | G(U-1) Q(U-2) | Q(U-1)
                int gu_entry = -1, gu_tile = 0;
                if (r < g.n_gu) {
                    gu_entry = 0;
                    gu_tile = r;
                } else if (r < U * g.n_gu + U) {
                    const int r2 = r - g.n_gu, b = 1 + r2 / (g.n_gu + 1), pos = r2 % (g.n_gu + 1);
                    if (b < U && pos < g.n_gu) {
                        gu_entry = b;
                        gu_tile = pos;
                    } else {
                        entry = 1 + (b - 1);  // QUANTISE of routed entry b-1
                    }
                }
                if (gu_entry >= 0) {
                    m.kind = kItemGateUp;
                    m.entry = 1 + gu_entry;
                    entry_tokens(m, m.entry);
                    m.row0 = gu_tile * g.rg;
                    m.nrows = g.rg;
                    src0 = p.routed.w_gate + ((int64_t)m.expert * p.I + m.row0) * rowH;
                    src1 = p.routed.w_up + ((int64_t)m.expert * p.I + m.row0) * rowH;
                    by0 = by1 = (uint32_t)(g.rg * rowH);
                    dof1 = by0;
                    src2 = p.routed.s_gate + (int64_t)m.expert * p.I + m.row0;
                    src3 = p.routed.s_up + (int64_t)m.expert * p.I + m.row0;
                    by2 = by3 = (uint32_t)(g.rg * 4);
                    dof2 = kSlotWeightBytes;
                    dof3 = kSlotWeightBytes + 64;
                    ncopy = 4;
                } else if (entry >= 1) {
                    // handled below (QUANTISE)
                } else {
                    r -= U * g.n_gu + U;  // past the gate/up + QUANTISE region
                    int down_entry = -1, tile = -1;
                    if (p.ns && r < g.n_dn) {
                        down_entry = 0;
                        tile = r;
                    } else {
                        if (p.ns) r -= g.n_dn;
                        if (r < U * g.n_dn) {
                            down_entry = 1 + r / g.n_dn;
                            tile = r % g.n_dn;
                        } else if ((r -= U * g.n_dn) < g.n_dn) {
                            // COMBINE of tile r
                            if (!wait_geq(p.ctrl + kCHeader + 2 * g.nent + r, (U + p.ns) * kWarpSignals))
                                return finish();
                            m.kind = kItemCombine;
                            m.row0 = r * g.rd;
                            m.nrows = (p.H - m.row0) < g.rd ? (p.H - m.row0) : g.rd;
                            combine_copies = true;
                        }
                    }
                    if (tile >= 0) {
                        if (!wait_hq(down_entry)) return finish();
                        m.kind = kItemDown;
                        m.entry = down_entry;
                        entry_tokens(m, down_entry);
                        m.row0 = tile * g.rd;
                        m.nrows = (p.H - m.row0) < g.rd ? (p.H - m.row0) : g.rd;
                        const moe_experts& ex = down_entry ? p.routed : p.shared;
                        const int eo = down_entry ? m.expert : 0;
                        src0 = ex.w_down + ((int64_t)eo * p.H + m.row0) * rowI;
                        by0 = (uint32_t)(m.nrows * rowI);
                        src1 = p.hq + (int64_t)m.slot0 * p.I;  // h codes (contiguous slots)
                        by1 = (uint32_t)(m.n * p.I);
                        dof1 = kSlotWeightBytes;
                        // h scales: a 16-byte aligned window covering the rows
                        const int nbI = p.I / 32;
                        const uintptr_t lo = reinterpret_cast<uintptr_t>(p.hd + (int64_t)m.slot0 * nbI);
                        const uintptr_t hi = reinterpret_cast<uintptr_t>(p.hd + (int64_t)(m.slot0 + m.n) * nbI);
                        const uintptr_t alo = lo & ~uintptr_t(15), ahi = (hi + 15) & ~uintptr_t(15);
                        src2 = reinterpret_cast<const void*>(alo);
                        by2 = (uint32_t)(ahi - alo);
                        dof2 = kSlotWeightBytes + round_up_dev(g.tmax * p.I, 16);
                        m.aux = (int)(dof2 - kSlotWeightBytes) + (int)(lo - alo);
                        // row scales of the down rows, after the h scales
                        src3 = ex.s_down + (int64_t)eo * p.H + m.row0;
                        by3 = (uint32_t)(m.nrows * 4);
                        dof3 = (uint32_t)(g.act_bytes - 64 * 4) + kSlotWeightBytes;
                        ncopy = 4;
                        if (m.n == 0) by1 = by2 = 0;
                    }
                }
            }
            if (entry >= 0) {
                // QUANTISE: wait for every gate/up item of the entry, then
                // bring its h rows (fp32) into the slot
                if (!wait_geq(p.ctrl + kCHeader + entry, g.n_gu * kWarpSignals)) return finish();
                if (entry > 0 && !know_routing()) return finish();
                m.kind = kItemQuant;
                m.entry = entry;
                entry_tokens(m, entry);
                src0 = p.hbuf + (int64_t)m.slot0 * p.I;
                by0 = (uint32_t)(m.n * p.I * 4);
                ncopy = 1;
            }
        }
        // ------------------------- hand the item over -------------------------
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&s.empty[slot], pe, kWaitLimit);
        ok = __shfl_sync(kFull, (int)ok, 0) != 0;
        if (!ok) {
            fail();
            return false;
        }
        uint8_t* dst = s.slots + (size_t)slot * g.slot_bytes;
        const int ns_slots = p.T * p.k + p.T * p.ns;
        const uint32_t rb = (uint32_t)m.nrows * 4;
        if (lane == 0) {
            s.meta[slot] = m;
            uint32_t total = (ncopy > 0 ? by0 : 0u) + (ncopy > 1 ? by1 : 0u) + (ncopy > 2 ? by2 : 0u) +
                             (ncopy > 3 ? by3 : 0u);
            if (combine_copies) total = (uint32_t)ns_slots * rb + 2u * (uint32_t)g.tk_pad * 4u;
            if (total == 0) mbar_arrive(&s.full[slot]);
            else mbar_arrive_expect_tx(&s.full[slot], total);
        }
        __syncwarp();
        // the copies go out from several lanes at once
        if (need_proxy_fence && lane < 32) fence_proxy_async_global();
        if (combine_copies) {
            for (int sl = lane; sl < ns_slots; sl += 32)
                bulk_g2s_nohint(dst + (size_t)sl * rb, p.y + (int64_t)sl * p.H + m.row0, rb, &s.full[slot]);
            if (lane == 31)
                bulk_g2s_nohint(dst + (size_t)ns_slots * rb, p.sched + g.sched_w_off, (uint32_t)g.tk_pad * 8u,
                                &s.full[slot]);
        } else if (lane < ncopy) {
            const void* sp = lane == 0 ? src0 : lane == 1 ? src1 : lane == 2 ? src2 : src3;
            const uint32_t bb = lane == 0 ? by0 : lane == 1 ? by1 : lane == 2 ? by2 : by3;
            const uint32_t dd = lane == 0 ? dof0 : lane == 1 ? dof1 : lane == 2 ? dof2 : dof3;
            if (bb) bulk_g2s(dst + dd, sp, bb, &s.full[slot], pol);
        }
        __syncwarp();
        need_proxy_fence = false;
        mark_issued();
        advance();
        return m.kind != kItemDone;
    }

    // After a timeout: hand the consumers a DONE marker if a slot frees up in
    // time (otherwise they time out on their own), and stop issuing.
    __forceinline__ __device__ bool finish() {
        int ok = 0;
        if (lane == 0 && mbar_wait(&s.empty[slot], pe, kWaitLimit)) {
            s.meta[slot].kind = kItemDone;
            mbar_arrive(&s.full[slot]);
            ok = 1;
        }
        ok = __shfl_sync(kFull, ok, 0);
        if (ok) {
            mark_issued();
            advance();
        }
        aborted = true;
        return false;
    }

    // Before the CTA exits: wait (bounded) for every copy it issued.
    __forceinline__ __device__ void drain() {
        if (lane != 0) return;
        for (int i = 0; i < p.g.nslot; ++i)
            if ((issued_mask >> i) & 1u) mbar_wait(&s.full[i], (issued_par >> i) & 1u, kWaitLimit);
    }
};

// ---------------------------------------------------------------------------
// Consumer helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void consumers_sync() { named_barrier(1, kConsumers); }

// SELECT: wait for every router item, then route all tokens and bucket them;
// publish the schedule record and raise the routing flag.  Same decisions as
// the multi-kernel router and the reference (group score = two largest c,
// keep topk_groups groups, then top_k experts in descending c, ties to the
// lower index, w = s / sum(s) * rsf).  Every decision is a rank: each thread
// owns one (token, expert) and counts the candidates that beat it, so there
// are no serial argmax rounds; the item's own ring slot is the scratch.
__device__ __forceinline__ bool beats(unsigned long long ka, int ia, unsigned long long kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

__device__ __forceinline__ void do_select(const SmallParams& p, SmemPtrs& s, uint8_t* scratch, int tid) {
    const int E = p.E, T = p.T, k = p.k, G = p.G, per = E / G;
    const int TE = T * E;
    double* sc = reinterpret_cast<double*>(scratch);                         // [T][E] c = s + bias
    double* ss = sc + TE;                                                     // [T][E] s
    unsigned long long* key = reinterpret_cast<unsigned long long*>(ss + TE);  // [T][E] order key of c
    unsigned long long* gkey = key + TE;                                      // [T][32] group-score keys
    int* top1 = reinterpret_cast<int*>(gkey + 4 * 32);                        // [T][32]
    int* top2 = top1 + 4 * 32;                                                // [T][32]
    int* kept = top2 + 4 * 32;                                                // [T][32]
    int* sel = kept + 4 * 32;                                                 // [T][32] picks, by rank
    int* cnt = sel + 4 * 32;                                                  // [E]
    int* off = cnt + 256;                                                     // [E] exclusive scan of counts
    int* ent = off + 256;                                                     // [E] entry index
    int* wsum = ent + 256;                                                    // [8][2] warp totals
    const int warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        int ok = 0;
        for (uint32_t i = 0; i < kSpinLimit; ++i) {
            if (ld_acquire_gpu(p.ctrl + kCRouterDone) >= p.g.n_router) {
                ok = 1;
                break;
            }
            __nanosleep(64);
        }
        if (!ok) set_error(p.err, kErrTimeout);  // route on whatever is there; never hang
    }
    consumers_sync();
    for (int i = tid; i < TE; i += kConsumers) {
        const double l = __ldcg(p.logits + i);
        const double sv = 1.0 / (1.0 + exp(-l));
        const double cv = sv + (double)p.bias[i % E];
        ss[i] = sv;
        sc[i] = cv;
        key[i] = order_key(cv);
    }
    for (int e = tid; e < E; e += kConsumers) cnt[e] = 0;
    consumers_sync();
    // group top-2: rank of each expert inside its group
    for (int i = tid; i < TE; i += kConsumers) {
        const int t = i / E, e = i - t * E, g = e / per;
        const unsigned long long* kt = key + (size_t)t * E;
        const unsigned long long ke = kt[e];
        int rank = 0;
        for (int e2 = g * per; e2 < (g + 1) * per; ++e2) rank += beats(kt[e2], e2, ke, e) ? 1 : 0;
        if (rank == 0) top1[t * 32 + g] = e;
        if (rank == 1) top2[t * 32 + g] = e;
    }
    consumers_sync();
    if (tid < T * 32) {
        const int t = tid >> 5, g = tid & 31;
        if (g < G) gkey[t * 32 + g] = order_key(sc[(size_t)t * E + top1[t * 32 + g]] + sc[(size_t)t * E + top2[t * 32 + g]]);
    }
    consumers_sync();
    if (tid < T * 32) {
        const int t = tid >> 5, g = tid & 31;
        if (g < G) {
            const unsigned long long kg = gkey[t * 32 + g];
            int rank = 0;
            for (int g2 = 0; g2 < G; ++g2) rank += beats(gkey[t * 32 + g2], g2, kg, g) ? 1 : 0;
            kept[t * 32 + g] = rank < p.tg ? 1 : 0;
        }
    }
    consumers_sync();
    // top_k experts of the kept groups: rank among the kept experts
    for (int i = tid; i < TE; i += kConsumers) {
        const int t = i / E, e = i - t * E;
        if (!kept[t * 32 + e / per]) continue;
        const unsigned long long* kt = key + (size_t)t * E;
        const unsigned long long ke = kt[e];
        int rank = 0;
        for (int g2 = 0; g2 < G; ++g2) {
            if (!kept[t * 32 + g2]) continue;
            for (int e2 = g2 * per; e2 < (g2 + 1) * per; ++e2) rank += beats(kt[e2], e2, ke, e) ? 1 : 0;
        }
        if (rank < k) sel[t * 32 + rank] = e;
    }
    consumers_sync();
    // weights from the unbiased sigmoid, summed in pick order
    if (warp < T && lane < k) {
        const int t = warp;
        double ssum = 0.0;
        for (int j = 0; j < k; ++j) ssum += ss[(size_t)t * E + sel[t * 32 + j]];
        const int e = sel[t * 32 + lane];
        const float wv = (float)(ss[(size_t)t * E + e] / ssum * (double)p.rsf);
        p.idx[(int64_t)t * k + lane] = e;
        p.w[(int64_t)t * k + lane] = wv;
        reinterpret_cast<float*>(p.sched + p.g.sched_w_off)[t * k + lane] = wv;
    }
    consumers_sync();
    const int n = T * k;
    if (tid < n) atomicAdd(&cnt[sel[(tid / k) * 32 + tid % k]], 1);
    consumers_sync();
    // block-wide exclusive scans over experts (one thread per expert, E <= 256)
    {
        const int cv = tid < E ? cnt[tid] : 0, nz = cv > 0 ? 1 : 0;
        int a1 = cv, a2 = nz;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u1 = __shfl_up_sync(kFull, a1, o), u2 = __shfl_up_sync(kFull, a2, o);
            if (lane >= o) {
                a1 += u1;
                a2 += u2;
            }
        }
        if (lane == 31) {
            wsum[warp * 2] = a1;
            wsum[warp * 2 + 1] = a2;
        }
        consumers_sync();
        int b1 = 0, b2 = 0;
        for (int w = 0; w < warp; ++w) {
            b1 += wsum[w * 2];
            b2 += wsum[w * 2 + 1];
        }
        if (tid < E) {
            const int o = b1 + a1 - cv, ai = b2 + a2 - nz;
            off[tid] = o;
            ent[tid] = ai;
            p.offsets[tid] = o;
            p.counts[tid] = cv;
            if (cv > 0) {
                int* r = p.sched + 1 + 8 * ai;  // schedule record of routed entry ai
                r[0] = tid;
                r[1] = o;
                r[2] = cv;
                p.active[1 + ai] = tid;
            }
            if (tid == E - 1) {
                p.offsets[E] = o + cv;
                p.active[0] = ai + nz;
                p.sched[0] = ai + nz;
            }
        }
    }
    consumers_sync();
    if (tid < n) {
        const int t = tid / k;
        const int e = sel[t * 32 + tid % k];
        int rank = 0;
        for (int t2 = 0; t2 < t; ++t2)
            for (int j2 = 0; j2 < k; ++j2) rank += sel[t2 * 32 + j2] == e ? 1 : 0;
        const int pos = off[e] + rank;
        p.perm[pos] = tid;
        p.inv_perm[tid] = pos;
        (p.sched + p.g.sched_w_off + p.g.tk_pad)[tid] = pos;
        if (rank < 4) p.sched[1 + 8 * ent[e] + 3 + rank] = t;
    }
    consumers_sync();  // every schedule write is done
    if (tid == 0) st_release_gpu(p.ctrl + kCRouting, 1);
}

// ---- router item: logits of two experts for all tokens ----
// Each lane accumulates its products with the compensated fp32 pair (about
// 2^-48 relative), the warps' partials are combined in fp64 in a fixed order.
// Uses shared scratch across warps, so it synchronises the consumer warps.
template <int TM>
__device__ __forceinline__ void do_router(const SmallParams& p, SmemPtrs& s, const SlotMeta& m, const uint8_t* slot, int tid,
                          uint64_t* empty) {
    const int warp = tid >> 5, lane = tid & 31;
    const int el = warp >> 2, qq = warp & 3;
    DFAcc acc[TM];
    if (el < m.nrows) {
        const float4* wr = reinterpret_cast<const float4*>(slot) + (size_t)el * (p.H / 4);
        const int nq = p.H / 16;
        // 4 float4 per lane per step, all loads issued before the arithmetic
        for (int j0 = qq * nq + lane; j0 < (qq + 1) * nq; j0 += 4 * 32) {
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                if (t < p.T) {
                    const float4* xr = reinterpret_cast<const float4*>(p.x + (int64_t)t * p.H);
                    float4 xv[4], wv[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int j = j0 + 32 * u;
                        const bool ok = j < (qq + 1) * nq;
                        xv[u] = ok ? __ldg(xr + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                        wv[u] = ok ? wr[j] : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        acc[t].add_prod(xv[u].x, wv[u].x);
                        acc[t].add_prod(xv[u].y, wv[u].y);
                        acc[t].add_prod(xv[u].z, wv[u].z);
                        acc[t].add_prod(xv[u].w, wv[u].w);
                    }
                }
            }
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty);
#pragma unroll
    for (int t = 0; t < TM; ++t) {
        double v = acc[t].value();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
        if (lane == 0) s.rpart[(el * 4 + qq) * 4 + t] = v;
    }
    consumers_sync();
    if (tid < m.nrows * p.T) {
        const int e2 = tid / p.T, t = tid % p.T;
        double v = 0.0;
#pragma unroll
        for (int k = 0; k < 4; ++k) v += s.rpart[(e2 * 4 + k) * 4 + t];
        p.logits[(int64_t)t * p.E + m.expert + e2] = v;
    }
    consumers_sync();  // logits written; rpart free for the next item
    if (tid == 0) red_add_release_gpu(p.ctrl + kCRouterDone, 1);
}

// Completion signals of one consumer warp, published in batches: the warp's
// global writes are ordered before one fence, then every pending counter gets
// a relaxed add (a release pattern).  The batch is flushed every few items and
// always before the warp could block, so no other item ever waits on a
// signal that is still held back.
struct Signals {
    int* p0 = nullptr;
    int* p1 = nullptr;
    int c0 = 0, c1 = 0;
    int age = 0;
    __device__ __forceinline__ void flush(int lane) {
        if (!p0) return;
        __syncwarp();
        if (lane == 0) {
            fence_acq_rel_gpu();
            red_add_relaxed_gpu(p0, c0);
            if (p1) red_add_relaxed_gpu(p1, c1);
        }
        __syncwarp();
        p0 = p1 = nullptr;
        c0 = c1 = 0;
        age = 0;
    }
    __device__ __forceinline__ void add(int* c, int lane) {
        if (p1 == c) {
            ++c1;
        } else if (!p1 && p0 == c) {
            ++c0;
        } else if (!p0) {
            p0 = c;
            c0 = 1;
        } else if (!p1) {
            p1 = c;
            c1 = 1;
        } else {
            flush(lane);
            p0 = c;
            c0 = 1;
        }
        if (++age >= 4) flush(lane);
    }
};

// ---- gate/up item: rg rows of Wg and Wu for the entry's tokens -> h ----
template <int WBITS, int TM>
__device__ __forceinline__ void do_gateup(const SmallParams& p, SmemPtrs& s, const SlotMeta& m, const uint8_t* slot, int tid,
                          uint64_t* empty, Signals& sig) {
    constexpr int V = 2 * TM;
    constexpr int SHIFT = 5 - Log2<V>::value;
    const int warp = tid >> 5, lane = tid & 31;
    const SmallGeom& g = p.g;
    const int pair = warp % g.rg, half = warp / g.rg;
    const int nb = p.H / 32;
    const int per_half = (nb + g.ks - 1) / g.ks;
    const int b_lo = half * per_half, b_hi = min(nb, b_lo + per_half);
    const int64_t rbH = (int64_t)p.H * WBITS / 8;
    const uint8_t* wg = slot + (size_t)pair * rbH;
    const uint8_t* wu = slot + (size_t)(g.rg + pair) * rbH;
    const float* sg = reinterpret_cast<const float*>(slot + kSlotWeightBytes);
    const float* su = reinterpret_cast<const float*>(slot + kSlotWeightBytes + 64);
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.0f;
    for (int b = b_lo + lane; b < b_hi; b += 32) {
        WBlock<WBITS> bg, bu;
        if constexpr (WBITS == 4) {
            bg.a = *reinterpret_cast<const uint4*>(wg + 16 * b);
            bu.a = *reinterpret_cast<const uint4*>(wu + 16 * b);
        } else {
            bg.a = *reinterpret_cast<const uint4*>(wg + 32 * b);
            bg.b = *reinterpret_cast<const uint4*>(wg + 32 * b + 16);
            bu.a = *reinterpret_cast<const uint4*>(wu + 32 * b);
            bu.b = *reinterpret_cast<const uint4*>(wu + 32 * b + 16);
        }
#pragma unroll
        for (int i = 0; i < TM; ++i) {
            if (i < m.n) {
                const int t = m.tok[i];
                const uint4 lo = *reinterpret_cast<const uint4*>(s.xq + ((size_t)(t * 2 + 0) * nb + b) * 16);
                const uint4 hi = *reinterpret_cast<const uint4*>(s.xq + ((size_t)(t * 2 + 1) * nb + b) * 16);
                ActBlock a;
                if constexpr (WBITS == 4) a = act_nibble_order(lo, hi);
                else a = act_natural(lo, hi);
                const float dx = s.xd[t * nb + b];
                acc[i] = fmaf(dx, (float)dot_block<WBITS>(bg, a), acc[i]);
                acc[TM + i] = fmaf(dx, (float)dot_block<WBITS>(bu, a), acc[TM + i]);
            }
        }
    }
    const float v = warp_reduce_many<V>(acc, lane);
    const float vu = __shfl_down_sync(kFull, v, 16);
    const int vi = lane >> SHIFT;
    const bool rep = lane < 16 && (lane & ((1 << SHIFT) - 1)) == 0;  // one lane per (g, token)
    int* counter = p.ctrl + kCHeader + m.entry;
    if (g.ks == 1) {
        const float sgv = sg[pair], suv = su[pair];
        __syncwarp();
        if (lane == 0) mbar_arrive(empty);
        if (rep && vi < m.n) {
            const float gv = sgv * v, uv = suv * vu;
            p.hbuf[(int64_t)(m.slot0 + vi) * p.I + m.row0 + pair] = silu_mul(gv, uv);
        }
        sig.add(counter, lane);
    } else {
        if (rep) {
            s.gpart[(pair * 2 + half) * 8 + vi] = v;
            s.gpart[(pair * 2 + half) * 8 + 4 + vi] = vu;
        }
        consumers_sync();
        if (tid < g.rg * TM) {
            const int pr = tid / TM, i = tid % TM;
            if (i < m.n) {
                const float gsum = s.gpart[(pr * 2) * 8 + i] + s.gpart[(pr * 2 + 1) * 8 + i];
                const float usum = s.gpart[(pr * 2) * 8 + 4 + i] + s.gpart[(pr * 2 + 1) * 8 + 4 + i];
                p.hbuf[(int64_t)(m.slot0 + i) * p.I + m.row0 + pr] = silu_mul(sg[pr] * gsum, su[pr] * usum);
            }
        }
        consumers_sync();  // h written by the first warp; gpart free for the next item
        __syncwarp();
        if (lane == 0) mbar_arrive(empty);
        sig.add(counter, lane);
    }
}

// ---- QUANTISE: Q8_0 of an entry's h rows (in the slot), published ----
__device__ __forceinline__ void do_quant(const SmallParams& p, const SlotMeta& m, const uint8_t* slot, int tid, uint64_t* empty,
                         Signals& sig) {
    const int warp = tid >> 5, lane = tid & 31;
    const int nbI = p.I / 32;
    const float* h = reinterpret_cast<const float*>(slot);
    for (int job = warp; job < m.n * nbI; job += kConsumerWarps) {
        const int i = job / nbI, bb = job % nbI;
        int8_t q;
        float d;
        q8_0_warp(h[(size_t)i * p.I + bb * 32 + lane], q, d);
        const int64_t sl = m.slot0 + i;
        p.hq[sl * p.I + bb * 32 + lane] = q;
        if (lane == 0) p.hd[sl * nbI + bb] = d;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty);
    sig.add(p.ctrl + kCHeader + p.g.nent + m.entry, lane);
    sig.flush(lane);  // a whole expert's down items wait for this one
}

// ---- down item: rd rows of Wd for the entry's tokens -> y ----
template <int WBITS, int TM>
__device__ __forceinline__ void do_down(const SmallParams& p, const SlotMeta& m, const uint8_t* slot, int tid, uint64_t* empty,
                        Signals& sig) {
    constexpr int V = 8 * TM;
    constexpr int SHIFT = 5 - Log2<V>::value;
    const int warp = tid >> 5, lane = tid & 31;
    const SmallGeom& g = p.g;
    const int nbI = p.I / 32;
    const int64_t rbI = (int64_t)p.I * WBITS / 8;
    const uint8_t* act = slot + kSlotWeightBytes;
    const float* hdv = reinterpret_cast<const float*>(act + m.aux);
    const float* sdv = reinterpret_cast<const float*>(act + g.act_bytes - 64 * 4);
    const int rpw = g.rd / 8;
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.0f;
    for (int b = lane; b < nbI; b += 32) {
        ActBlock a[TM];
        float dh[TM];
#pragma unroll
        for (int i = 0; i < TM; ++i) {
            if (i < m.n) {
                const uint4 lo = *reinterpret_cast<const uint4*>(act + (size_t)i * p.I + 32 * b);
                const uint4 hi = *reinterpret_cast<const uint4*>(act + (size_t)i * p.I + 32 * b + 16);
                if constexpr (WBITS == 4) a[i] = act_nibble_order(lo, hi);
                else a[i] = act_natural(lo, hi);
                dh[i] = hdv[i * nbI + b];
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = warp + 8 * j;
            if (j < rpw && r < m.nrows) {
                const uint8_t* row = slot + (size_t)r * rbI;
                WBlock<WBITS> wb;
                if constexpr (WBITS == 4) {
                    wb.a = *reinterpret_cast<const uint4*>(row + 16 * b);
                } else {
                    wb.a = *reinterpret_cast<const uint4*>(row + 32 * b);
                    wb.b = *reinterpret_cast<const uint4*>(row + 32 * b + 16);
                }
#pragma unroll
                for (int i = 0; i < TM; ++i)
                    if (i < m.n) acc[j * TM + i] = fmaf(dh[i], (float)dot_block<WBITS>(wb, a[i]), acc[j * TM + i]);
            }
        }
    }
    const float v = warp_reduce_many<V>(acc, lane);
    const int vi = lane >> SHIFT;
    const int j = vi / TM, i = vi % TM;
    const int r = warp + 8 * j;
    const bool mine = (lane & ((1 << SHIFT) - 1)) == 0 && j < rpw && r < m.nrows && i < m.n;
    const float sd = mine ? sdv[r] : 0.0f;
    __syncwarp();
    if (lane == 0) mbar_arrive(empty);
    if (mine) p.y[(int64_t)(m.slot0 + i) * p.H + m.row0 + r] = sd * v;
    sig.add(p.ctrl + kCHeader + 2 * g.nent + m.row0 / g.rd, lane);
}

// ---- COMBINE: out rows of one tile from every slot's y (in the slot) ----
__device__ __forceinline__ void do_combine(const SmallParams& p, const SlotMeta& m, const uint8_t* slot, int tid, uint64_t* empty) {
    const int rows = m.nrows;
    const int ns_slots = p.T * p.k + p.T * p.ns;
    const float* ys = reinterpret_cast<const float*>(slot);
    const float* wv = ys + (size_t)ns_slots * rows;
    const int* inv = reinterpret_cast<const int*>(wv + p.g.tk_pad);
    for (int idx = tid; idx < p.T * rows; idx += kConsumers) {
        const int t = idx / rows, r = idx % rows;
        float acc = 0.0f;  // fixed order: slots 0..k-1, then the shared expert
        for (int j = 0; j < p.k; ++j) {
            int sl = inv[t * p.k + j];
            sl = (sl < 0 || sl >= p.T * p.k) ? 0 : sl;
            acc = fmaf(wv[t * p.k + j], ys[(size_t)sl * rows + r], acc);
        }
        if (p.ns) acc += ys[(size_t)(p.T * p.k + t) * rows + r];
        p.out[(int64_t)t * p.H + m.row0 + r] = acc;
    }
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(empty);
}

// ---------------------------------------------------------------------------
// Main kernel
// ---------------------------------------------------------------------------
template <int WBITS, int TM>
__global__ void __launch_bounds__(kSmallThreads, 1) k_moe_small(const __grid_constant__ SmallParams p) {
    extern __shared__ __align__(128) uint8_t smem_raw[];
    SmemPtrs s = carve(smem_raw, p.g, p.H);
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < p.g.nslot; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], kConsumerWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------- producer -------------------------
        Producer pr(p, s, lane);
        // the first item depends on nothing from the prologue
        if (p.g.n_static) pr.issue(blockIdx.x);
        pdl_wait();
        const int base = p.g.n_static * gridDim.x;
        // two consecutive items per queue atomic; the next batch index is
        // requested one batch ahead so its round trip overlaps the issue
        int pending = 0;
        if (lane == 0) pending = atom_add_relaxed_gpu(p.ctrl + kCQueue, 1);
        while (true) {
            const int q = base + 2 * __shfl_sync(kFull, pending, 0);
            if (lane == 0) pending = atom_add_relaxed_gpu(p.ctrl + kCQueue, 1);
            if (!pr.issue(q)) break;
            if (!pr.issue(q + 1)) break;
        }
        pr.drain();
        return;
    }

    // ------------------------- consumers -------------------------
    pdl_wait();
    {
        // Q8_0 activations of all tokens into shared memory, each 32-code
        // block split in 16-byte halves so that lanes read consecutive words
        const int nb = p.H / 32;
        for (int job = tid; job < p.T * nb * 2; job += kConsumers) {
            const int t = job / (2 * nb), rem = job % (2 * nb), half = rem / nb, b = rem % nb;
            const uint4 v = __ldcg(reinterpret_cast<const uint4*>(p.xq + (int64_t)t * p.H + b * 32 + half * 16));
            *reinterpret_cast<uint4*>(s.xq + ((size_t)(t * 2 + half) * nb + b) * 16) = v;
        }
        for (int job = tid; job < p.T * nb; job += kConsumers) s.xd[job] = __ldcg(p.xd + job);
    }
    consumers_sync();
    // Every consumer warp walks the ring on its own; only items that combine
    // partial results across warps (router, select, int8 gate/up) synchronise.
    int slot = 0;
    uint32_t pf = 0;
    Signals sig;
    while (true) {
        if (!mbar_try_wait(&s.full[slot], pf)) {
            sig.flush(lane);  // about to block: publish what this warp has done
            if (!mbar_wait(&s.full[slot], pf, kConsumerWaitLimit)) {
                set_error(p.err, kErrTimeout);
                break;
            }
        }
        const SlotMeta m = s.meta[slot];
        const uint8_t* data = s.slots + (size_t)slot * p.g.slot_bytes;
        uint64_t* empty = &s.empty[slot];
        if (m.kind == kItemGateUp) {
            if (p.g.ks != 1) sig.flush(lane);  // this item synchronises the warps
            do_gateup<WBITS, TM>(p, s, m, data, tid, empty, sig);
        } else if (m.kind == kItemDown) {
            do_down<WBITS, TM>(p, m, data, tid, empty, sig);
        } else if (m.kind == kItemRouter) {
            sig.flush(lane);
            do_router<TM>(p, s, m, data, tid, empty);
        } else if (m.kind == kItemQuant) {
            do_quant(p, m, data, tid, empty, sig);
        } else if (m.kind == kItemCombine) {
            do_combine(p, m, data, tid, empty);
        } else if (m.kind == kItemSelect) {
            sig.flush(lane);
            do_select(p, s, const_cast<uint8_t*>(data), tid);
            __syncwarp();
            if (lane == 0) mbar_arrive(empty);  // the slot was the scratch
        } else {
            break;  // DONE (or an unknown marker)
        }
        if (++slot == p.g.nslot) {
            slot = 0;
            pf ^= 1u;
        }
    }
    sig.flush(lane);
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------
template <int WBITS, int TM>
static cudaError_t launch_small_t(const SmallParams& prm, cudaStream_t st) {
    static bool attr_done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(k_moe_small<WBITS, TM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             device_info().max_smem_optin);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(device_info().sm_count);
    cfg.blockDim = dim3(kSmallThreads);
    cfg.dynamicSmemBytes = prm.g.smem_bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_moe_small<WBITS, TM>, prm);
}

cudaError_t launch_small(const SmallArgs& a, cudaStream_t st) {
    const moe_config& c = *a.cfg;
    SmallParams p;
    p.T = a.T; p.H = c.hidden; p.I = c.inter; p.E = c.n_experts; p.G = c.n_groups; p.tg = c.topk_groups;
    p.k = c.top_k; p.ns = c.n_shared; p.wbits = c.wbits; p.rsf = c.routed_scaling_factor;
    p.x = a.x; p.router_w = a.router_w; p.bias = a.bias; p.routed = a.routed; p.shared = a.shared;
    p.xq = a.xq; p.xd = a.xd; p.logits = a.logits; p.idx = a.idx; p.w = a.w; p.counts = a.counts;
    p.offsets = a.offsets; p.perm = a.perm; p.inv_perm = a.inv_perm; p.active = a.active;
    p.hbuf = a.hbuf; p.hq = a.hq; p.hd = a.hd; p.y = a.y; p.out = a.out; p.ctrl = a.ctrl; p.err = a.err;
    p.g = small_geometry(c, a.T, device_info().sm_count);
    p.sched = a.ctrl + p.g.ctrl_words;
    if (p.g.smem_bytes > device_info().max_smem_optin) return cudaErrorInvalidConfiguration;
    const int64_t nblk = (int64_t)a.T * (c.hidden / 32);
    const int grid = (int)((nblk + 7) / 8) > 1 ? (int)((nblk + 7) / 8) : 1;
    k_small_prologue<<<grid, 256, 0, st>>>(a.x, nblk, a.xq, a.xd, a.ctrl, p.g.ctrl_words, a.err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int tm = p.g.tmax;
    if (c.wbits == 4) {
        if (tm == 1) return launch_small_t<4, 1>(p, st);
        if (tm == 2) return launch_small_t<4, 2>(p, st);
        return launch_small_t<4, 4>(p, st);
    }
    if (tm == 1) return launch_small_t<8, 1>(p, st);
    if (tm == 2) return launch_small_t<8, 2>(p, st);
    return launch_small_t<8, 4>(p, st);
}

}  // namespace moe
