// moe_expert.cu -- SwiGLU experts on Q8_0 activations (integer dots) and the
// weighted combine.
//
// GeekNews "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", §구현된 주요 기능: the expert
// matmuls multiply Q8_0-style int8 activations by int8 / packed int4 weights
// with per-row scales, dequantised on use; "Batch-union MoE" reads each unique
// expert once for all positions routed to it.  wpnews.pro "Colibri — รัน
// GLM-5.2 ...", kernel table (int4 packed, dequant-on-use, used for the expert
// matmul) and spec table (8 active + 1 shared).
//
// Work is split into items (expert, tile of rows).  Each item streams its rows
// from HBM exactly once with 128-bit loads and applies them to every token of
// the expert's bucket, a few tokens at a time from registers.  Inside a warp,
// lane l owns Q8_0 blocks l, l+32, ... of a row, so a warp load covers 512
// (int4) or 1024 (int8) contiguous bytes.
#include <cmath>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

struct ExpertParams {
    int T, H, I, E, k, ns;
    const int8_t* xq;
    const float* xd;
    const float* w;
    const int32_t* offsets;
    const int32_t* perm;
    const int32_t* inv_perm;
    const int32_t* active;
    moe_experts routed;
    moe_experts shared;
    int8_t* hq;
    float* hd;
    float* y;
    float* out;
    int32_t* err;
};

// Token list of work entry `entry`: routed entries are active experts (their
// bucket's slots), the entry after them is the shared expert (slot T*k + t).
struct Entry {
    int expert;    // -1 = shared
    int slot0;     // first slot
    int n;         // tokens
};

__device__ __forceinline__ Entry get_entry(const ExpertParams& p, int entry, int n_act) {
    Entry en;
    if (entry < n_act) {
        en.expert = p.active[1 + entry];
        en.slot0 = p.offsets[en.expert];
        en.n = p.offsets[en.expert + 1] - en.slot0;
    } else {
        en.expert = -1;
        en.slot0 = p.T * p.k;
        en.n = p.T;
    }
    return en;
}

__device__ __forceinline__ int slot_token(const ExpertParams& p, const Entry& en, int i) {
    return en.expert >= 0 ? p.perm[en.slot0 + i] / p.k : i;
}

// ---------------------------------------------------------------------------
// gate/up: item = (entry, 32-row tile).  Warp w owns rows 4w..4w+3 of the tile
// in both Wg and Wu (8 row dots).  After the K loop, h = silu(g) * u for the
// 32 rows is exactly one Q8_0 block of h per token, quantised in the CTA.
// ---------------------------------------------------------------------------
template <int WBITS, int TCH>
__global__ void __launch_bounds__(256) k_gateup(ExpertParams p) {
    constexpr int V = 8 * TCH;
    constexpr int SHIFT = 5 - Log2<V>::value;
    __shared__ float hs[TCH][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_act = p.active[0];
    const int tiles = p.I / 32;
    const int n_items = (n_act + p.ns) * tiles;
    const int nb = p.H / kQBlock;
    const int64_t rb = (int64_t)p.H * WBITS / 8;  // row bytes
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int entry = item / tiles, tile = item % tiles;
        const Entry en = get_entry(p, entry, n_act);
        const moe_experts& ex = en.expert >= 0 ? p.routed : p.shared;
        const int eo = en.expert >= 0 ? en.expert : 0;
        const int row0 = tile * 32 + warp * 4;
        const uint8_t* wg = ex.w_gate + ((int64_t)eo * p.I + row0) * rb;
        const uint8_t* wu = ex.w_up + ((int64_t)eo * p.I + row0) * rb;
        for (int c0 = 0; c0 < en.n; c0 += TCH) {
            const int nv = min(TCH, en.n - c0);
            int tok[TCH];
#pragma unroll
            for (int i = 0; i < TCH; ++i) tok[i] = i < nv ? slot_token(p, en, c0 + i) : 0;
            float acc[V];
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] = 0.0f;
            for (int b = lane; b < nb; b += 32) {
                WBlock<WBITS> wblk[8];
#pragma unroll
                for (int rd = 0; rd < 8; ++rd)
                    wblk[rd] = load_w_block<WBITS>((rd < 4 ? wg : wu) + (rd & 3) * rb, b);
#pragma unroll
                for (int i = 0; i < TCH; ++i) {
                    if (i < nv) {
                        const ActBlock a = load_act_block<WBITS>(p.xq + (int64_t)tok[i] * p.H + b * kQBlock);
                        const float dx = p.xd[(int64_t)tok[i] * nb + b];
#pragma unroll
                        for (int rd = 0; rd < 8; ++rd)
                            acc[rd * TCH + i] = fmaf(dx, (float)dot_block<WBITS>(wblk[rd], a), acc[rd * TCH + i]);
                    }
                }
            }
            const float v = warp_reduce_many<V>(acc, lane);
            const float vu = __shfl_down_sync(kFull, v, 16);
            const int vi = lane >> SHIFT;  // = rd * TCH + i
            if (lane < 16 && (lane & ((1 << SHIFT) - 1)) == 0) {
                const int rd = vi / TCH, i = vi % TCH;
                const int row = row0 + rd;
                const int64_t so = (int64_t)eo * p.I + row;
                hs[i][warp * 4 + rd] = silu_mul(ex.s_gate[so] * v, ex.s_up[so] * vu);
            }
            __syncthreads();
            if (warp < nv) {
                int8_t q;
                float d;
                q8_0_warp(hs[warp][lane], q, d);
                const int64_t slot = en.slot0 + c0 + warp;
                p.hq[slot * p.I + tile * 32 + lane] = q;
                if (lane == 0) p.hd[slot * (p.I / kQBlock) + tile] = d;
            }
            __syncthreads();
        }
    }
}

// ---------------------------------------------------------------------------
// down: item = (entry, 64-row tile of Wd [H][I]).  Warp w owns rows 8w..8w+7.
// y[slot][row] = s_down[row] * sum_b hd[slot][b] * isum_b(Wd[row], hq[slot]).
// ---------------------------------------------------------------------------
template <int WBITS, int TCH>
__global__ void __launch_bounds__(256) k_down(ExpertParams p) {
    constexpr int V = 8 * TCH;
    constexpr int SHIFT = 5 - Log2<V>::value;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_act = p.active[0];
    const int tiles = (p.H + 63) / 64;
    const int n_items = (n_act + p.ns) * tiles;
    const int nb = p.I / kQBlock;
    const int64_t rb = (int64_t)p.I * WBITS / 8;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int entry = item / tiles, tile = item % tiles;
        const Entry en = get_entry(p, entry, n_act);
        const moe_experts& ex = en.expert >= 0 ? p.routed : p.shared;
        const int eo = en.expert >= 0 ? en.expert : 0;
        const int row0 = tile * 64 + warp * 8;
        const int nrows = max(0, min(8, p.H - row0));
        const uint8_t* wd = ex.w_down + ((int64_t)eo * p.H + row0) * rb;
        for (int c0 = 0; c0 < en.n; c0 += TCH) {
            const int nv = min(TCH, en.n - c0);
            float acc[V];
#pragma unroll
            for (int i = 0; i < V; ++i) acc[i] = 0.0f;
            for (int b = lane; b < nb; b += 32) {
                WBlock<WBITS> wblk[8];
#pragma unroll
                for (int rd = 0; rd < 8; ++rd)
                    if (rd < nrows) wblk[rd] = load_w_block<WBITS>(wd + rd * rb, b);
#pragma unroll
                for (int i = 0; i < TCH; ++i) {
                    if (i < nv) {
                        const int64_t slot = en.slot0 + c0 + i;
                        const ActBlock a = load_act_block<WBITS>(p.hq + slot * p.I + b * kQBlock);
                        const float dh = p.hd[slot * nb + b];
#pragma unroll
                        for (int rd = 0; rd < 8; ++rd)
                            if (rd < nrows)
                                acc[rd * TCH + i] =
                                    fmaf(dh, (float)dot_block<WBITS>(wblk[rd], a), acc[rd * TCH + i]);
                    }
                }
            }
            const float v = warp_reduce_many<V>(acc, lane);
            const int vi = lane >> SHIFT;
            if ((lane & ((1 << SHIFT) - 1)) == 0) {
                const int rd = vi / TCH, i = vi % TCH;
                if (rd < nrows && i < nv) {
                    const int row = row0 + rd;
                    const int64_t slot = en.slot0 + c0 + i;
                    p.y[slot * p.H + row] = ex.s_down[(int64_t)eo * p.H + row] * v;
                }
            }
        }
    }
}

// out[t][c] = sum_j w[t][j] * y[slot(t,j)][c] + y[T*k + t][c], summed in
// fp64 in slot order, then the shared expert, and rounded to fp32 (each
// fp32 x fp32 product is exact in fp64, so every step rounds once, as the
// definition's fp64 sum does).  CTA = one token x kCombineCols columns: the
// token's slots and weights are read once into shared memory, each thread
// then streams four columns of every slot's row (128-bit loads).
constexpr int kCombineCols = 1024;
__global__ void __launch_bounds__(256) k_combine(ExpertParams p) {
    __shared__ int s_slot[33];
    __shared__ double s_w[33];
    const int t = blockIdx.y;
    const int k = p.k;
    if ((int)threadIdx.x < k) {
        s_slot[threadIdx.x] = p.inv_perm[t * k + threadIdx.x];  // < 0: dropped by the adaptive top-p
        s_w[threadIdx.x] = (double)p.w[t * k + threadIdx.x];
    }
    __syncthreads();
    const int c = blockIdx.x * kCombineCols + 4 * threadIdx.x;
    if (c >= p.H) return;
    double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
    for (int j = 0; j < k; ++j) {
        const int slot = s_slot[j];
        if (slot < 0) continue;
        const float4 y = __ldcs(reinterpret_cast<const float4*>(p.y + (int64_t)slot * p.H + c));
        const double w = s_w[j];
        a0 = __fma_rn(w, (double)y.x, a0);
        a1 = __fma_rn(w, (double)y.y, a1);
        a2 = __fma_rn(w, (double)y.z, a2);
        a3 = __fma_rn(w, (double)y.w, a3);
    }
    if (p.ns) {
        const float4 y = __ldcs(reinterpret_cast<const float4*>(p.y + ((int64_t)p.T * k + t) * p.H + c));
        a0 = __dadd_rn(a0, (double)y.x);
        a1 = __dadd_rn(a1, (double)y.y);
        a2 = __dadd_rn(a2, (double)y.z);
        a3 = __dadd_rn(a3, (double)y.w);
    }
    float* o = p.out + (int64_t)t * p.H + c;  // out is only 4-byte aligned
    o[0] = __double2float_rn(a0);
    o[1] = __double2float_rn(a1);
    o[2] = __double2float_rn(a2);
    o[3] = __double2float_rn(a3);
}

template <typename K>
static int ctas_per_sm(K kernel) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, 256, 0) != cudaSuccess || n < 1) n = 1;
    return n;
}

template <int WBITS, int TCH>
static cudaError_t launch_experts_t(const ExpertParams& p, cudaStream_t s, cudaEvent_t const* ev) {
    const DeviceInfo& di = device_info();
    const int max_entries = min(p.E, p.T * p.k) + p.ns;
    static const int occ_gu = ctas_per_sm(k_gateup<WBITS, TCH>);
    static const int occ_dn = ctas_per_sm(k_down<WBITS, TCH>);
    const int items_gu = max_entries * (p.I / 32);
    const int items_dn = max_entries * ((p.H + 63) / 64);
    k_gateup<WBITS, TCH><<<max(1, min(items_gu, di.sm_count * occ_gu)), 256, 0, s>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess && ev) e = record_event(ev[0], s);
    if (e != cudaSuccess) return e;
    k_down<WBITS, TCH><<<max(1, min(items_dn, di.sm_count * occ_dn)), 256, 0, s>>>(p);
    e = cudaGetLastError();
    if (e == cudaSuccess && ev) e = record_event(ev[1], s);
    if (e != cudaSuccess) return e;
    k_combine<<<dim3((p.H + kCombineCols - 1) / kCombineCols, p.T), 256, 0, s>>>(p);
    e = cudaGetLastError();
    if (e == cudaSuccess && ev) e = record_event(ev[2], s);
    return e;
}

static ExpertParams expert_params(const ExpertArgs& a) {
    const moe_config& c = *a.cfg;
    ExpertParams p;
    p.T = a.T; p.H = c.hidden; p.I = c.inter; p.E = c.n_experts; p.k = c.top_k; p.ns = c.n_shared;
    p.xq = a.xq; p.xd = a.xd; p.w = a.w; p.offsets = a.offsets; p.perm = a.perm; p.inv_perm = a.inv_perm;
    p.active = a.active; p.routed = a.routed; p.shared = a.shared;
    p.hq = a.hq; p.hd = a.hd; p.y = a.y; p.out = a.out; p.err = a.err;
    return p;
}

cudaError_t launch_combine(const ExpertArgs& a, cudaStream_t s) {
    const ExpertParams p = expert_params(a);
    if (p.T == 0) return cudaSuccess;
    const dim3 grid((p.H + kCombineCols - 1) / kCombineCols, p.T);
    k_combine<<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_experts(const ExpertArgs& a, cudaStream_t s, cudaEvent_t const* ev) {
    const moe_config& c = *a.cfg;
    ExpertParams p;
    p.T = a.T; p.H = c.hidden; p.I = c.inter; p.E = c.n_experts; p.k = c.top_k; p.ns = c.n_shared;
    p.xq = a.xq; p.xd = a.xd; p.w = a.w; p.offsets = a.offsets; p.perm = a.perm; p.inv_perm = a.inv_perm;
    p.active = a.active; p.routed = a.routed; p.shared = a.shared;
    p.hq = a.hq; p.hd = a.hd; p.y = a.y; p.out = a.out; p.err = a.err;
    const int tch = a.T == 1 ? 1 : a.T == 2 ? 2 : 4;
    if (c.wbits == 4) {
        if (tch == 1) return launch_experts_t<4, 1>(p, s, ev);
        if (tch == 2) return launch_experts_t<4, 2>(p, s, ev);
        return launch_experts_t<4, 4>(p, s, ev);
    }
    if (c.wbits == 2) {
        if (tch == 1) return launch_experts_t<2, 1>(p, s, ev);
        if (tch == 2) return launch_experts_t<2, 2>(p, s, ev);
        return launch_experts_t<2, 4>(p, s, ev);
    }
    if (tch == 1) return launch_experts_t<8, 1>(p, s, ev);
    if (tch == 2) return launch_experts_t<8, 2>(p, s, ev);
    return launch_experts_t<8, 4>(p, s, ev);
}

// ---------------------------------------------------------------------------
// Per-block dot export: one warp per (row, token), lane = block.
// ---------------------------------------------------------------------------
template <int WBITS>
__global__ void __launch_bounds__(256) k_block_dots(const uint8_t* __restrict__ packed, int64_t rows, int cols,
                                                    const int8_t* __restrict__ q, int n, int32_t* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (wid >= rows * n) return;
    const int64_t r = wid % rows, t = wid / rows;
    const int nb = cols / kQBlock;
    const uint8_t* row = packed + r * ((int64_t)cols * WBITS / 8);
    for (int b = lane; b < nb; b += 32) {
        const ActBlock a = load_act_block<WBITS>(q + t * cols + b * kQBlock);
        out[(t * rows + r) * nb + b] = dot_block<WBITS>(load_w_block<WBITS>(row, b), a);
    }
}

// The fused small-batch kernel's routine: the activation block is put in the
// weights' order by the same reordering (act_nibble_order / act_crumb_order),
// its correction term taken by act_corr, and the block dotted by
// dot_block_scaled, which returns the dot times dot_scale (16 for int4, 64 for
// int2, 1 for int8) exactly; that scaled value is what is stored.
template <int WBITS>
__global__ void __launch_bounds__(256) k_block_dots_fused(const uint8_t* __restrict__ packed, int64_t rows, int cols,
                                                          const int8_t* __restrict__ q, int n,
                                                          int32_t* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t wid = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (wid >= rows * n) return;
    const int64_t r = wid % rows, t = wid / rows;
    const int nb = cols / kQBlock;
    const uint8_t* row = packed + r * ((int64_t)cols * WBITS / 8);
    for (int b = lane; b < nb; b += 32) {
        const uint4 lo = ld_nc_v4(q + t * cols + b * kQBlock);
        const uint4 hi = ld_nc_v4(q + t * cols + b * kQBlock + 16);
        ActBlock a;
        if constexpr (WBITS == 4) a = act_nibble_order(lo, hi);
        else if constexpr (WBITS == 2) a = act_crumb_order(lo, hi);
        else a = act_natural(lo, hi);
        out[(t * rows + r) * nb + b] = dot_block_scaled<WBITS>(load_w_block<WBITS>(row, b), a, act_corr<WBITS>(a));
    }
}

cudaError_t launch_block_dots(const uint8_t* packed, int64_t rows, int cols, int wbits, const int8_t* q, int n,
                              int32_t* out, cudaStream_t s, int routine) {
    const int64_t warps = rows * n;
    if (warps == 0) return cudaSuccess;
    const int64_t grid = (warps + 7) / 8;
    if (grid > 0x7fffffff) return cudaErrorInvalidValue;
    if (routine == MOE_DOTS_FUSED) {
        if (wbits == 4) k_block_dots_fused<4><<<(unsigned)grid, 256, 0, s>>>(packed, rows, cols, q, n, out);
        else if (wbits == 2) k_block_dots_fused<2><<<(unsigned)grid, 256, 0, s>>>(packed, rows, cols, q, n, out);
        else k_block_dots_fused<8><<<(unsigned)grid, 256, 0, s>>>(packed, rows, cols, q, n, out);
        return cudaGetLastError();
    }
    if (wbits == 4) k_block_dots<4><<<(unsigned)grid, 256, 0, s>>>(packed, rows, cols, q, n, out);
    else if (wbits == 2) k_block_dots<2><<<(unsigned)grid, 256, 0, s>>>(packed, rows, cols, q, n, out);
    else k_block_dots<8><<<(unsigned)grid, 256, 0, s>>>(packed, rows, cols, q, n, out);
    return cudaGetLastError();
}

}  // namespace moe
