// moe_router.cu -- DeepSeek-V3-style sigmoid router with noaux_tc grouped top-k.
//
// GeekNews "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", §구현된 주요 기능 (sigmoid
// router, noaux_tc, routed_scaling_factor, shared expert); wpnews.pro "Colibri
// — รัน GLM-5.2 ...", spec table (Router: DeepSeek-V3-style sigmoid (noaux_tc);
// 256 experts, 8 active + 1 shared) and kernel table (the routing matmul stays
// in f32).  The logits keep fp32 inputs and are summed to about 2^-48
// relative (compensated fp32, then fp64) so that the expert choice does not
// depend on the summation order.
#include <cmath>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kRouterExpertsPerCta = 2;
constexpr int kRouterKSplit = 4;
constexpr int kRouterTokens = 8;

// logits[t][e] = sum_j x[t][j] * Wr[e][j], accumulated per lane with the
// compensated fp32 pair (about 2^-48 relative) and combined in fp64.  CTA = 2
// experts x 4 K-splits (one warp each) x up to 8 tokens; the K-split partials
// are added in a fixed order so the result is deterministic.
__global__ void __launch_bounds__(256) k_router_logits(const float* __restrict__ x, int T, int H,
                                                       const float* __restrict__ Wr, int E,
                                                       double* __restrict__ logits) {
    __shared__ double part[kRouterKSplit][kRouterExpertsPerCta][kRouterTokens];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int el = warp / kRouterKSplit, ks = warp % kRouterKSplit;
    const int e = blockIdx.x * kRouterExpertsPerCta + el;
    const int t0 = blockIdx.y * kRouterTokens;
    const int nt = min(kRouterTokens, T - t0);
    const int n4 = H / 4;
    const int per = (n4 + kRouterKSplit - 1) / kRouterKSplit;
    const int j0 = ks * per, j1 = min(n4, j0 + per);
    DFAcc acc[kRouterTokens];
    if (e < E) {
        const float4* wr = reinterpret_cast<const float4*>(Wr + (int64_t)e * H);
        for (int j = j0 + lane; j < j1; j += 32) {
            const float4 wv = __ldg(wr + j);
#pragma unroll
            for (int t = 0; t < kRouterTokens; ++t) {
                if (t < nt) {
                    const float4 xv = __ldg(reinterpret_cast<const float4*>(x + (int64_t)(t0 + t) * H) + j);
                    acc[t].add_prod(xv.x, wv.x);
                    acc[t].add_prod(xv.y, wv.y);
                    acc[t].add_prod(xv.z, wv.z);
                    acc[t].add_prod(xv.w, wv.w);
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < kRouterTokens; ++t) {
        double v = acc[t].value();
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
        if (lane == 0) part[ks][el][t] = v;
    }
    __syncthreads();
    if (threadIdx.x < kRouterExpertsPerCta * kRouterTokens) {
        const int el2 = threadIdx.x / kRouterTokens, t = threadIdx.x % kRouterTokens;
        const int e2 = blockIdx.x * kRouterExpertsPerCta + el2;
        if (e2 < E && t < nt) {
            double v = 0.0;
#pragma unroll
            for (int k = 0; k < kRouterKSplit; ++k) v += part[k][el2][t];
            logits[(int64_t)(t0 + t) * E + e2] = v;
        }
    }
}

// Batched logits (T >= kRouterTiledMinTokens): a tiled fp64 GEMM on the fp64
// tensor cores (mma.sync m8n8k4 .f64).  CTA = 64 tokens x 64 experts x one K
// split, 8 warps of 32 tokens x 16 experts (4 x 2 MMA tiles); x and the
// router rows are staged per 32-column chunk in shared memory, widened to
// fp64 (every fp32 product is then exact and every sum rounds in fp64, as
// the definition's), the next chunk's loads in flight during the MMAs.  The
// K splits' partial sums go to parts [S][T][E] and are added in split order
// by k_router_reduce, so the logits do not depend on the launch.  The split
// count aims at three CTAs on each of 148 SMs (the kernel is latency-bound:
// more resident warps, not fewer chunks, shorten it).
constexpr int kRtT = 64, kRtE = 64, kRtK = 32;
constexpr int kRtPad = 4;  // rows of 36 doubles: conflict-free fragment loads and staging stores
constexpr int kRtTargetCtas = 3 * 148;
constexpr int kRtMaxSplits = 48;  // a few tokens: a few tiles, split finely (parts: S x T x E doubles)

int router_splits(const moe_config& c, int T) {
    if (T < kRouterTiledMinTokens || c.hidden % kRtK) return 0;
    const int tiles = ((T + kRtT - 1) / kRtT) * ((c.n_experts + kRtE - 1) / kRtE);
    int want = kRtTargetCtas / tiles;  // never a second, partial wave
    want = want < 1 ? 1 : want > kRtMaxSplits ? kRtMaxSplits : want;
    const int chunks = c.hidden / kRtK;
    return want < chunks ? want : chunks;
}

// D += A (8 x 4) x B (4 x 8) in fp64 on one warp: lane l holds A[l / 4][l % 4],
// B[l % 4][l / 4] and D[l / 4][2 (l % 4) + j], j = 0, 1.
__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d[0]), "+d"(d[1])
                 : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(256) k_router_logits_f64(const float* __restrict__ x, int T, int H,
                                                           const float* __restrict__ Wr, int E, int chunks_per_split,
                                                           double* __restrict__ parts) {
    __shared__ __align__(16) double xs[kRtT][kRtK + kRtPad];  // [token][k]
    __shared__ __align__(16) double ws[kRtE][kRtK + kRtPad];  // [expert][k]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, q = lane & 3;
    const int t0 = blockIdx.y * kRtT, e0 = blockIdx.x * kRtE, split = blockIdx.z;
    const int wt = (warp & 1) * 32, we = (warp >> 1) * 16;  // the warp's tokens and experts in the tile
    const int nchunks = H / kRtK;
    const int kc0 = split * chunks_per_split;
    const int kc1 = min(nchunks, kc0 + chunks_per_split);
    double acc[4][2][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 2; ++c) acc[i][c][0] = acc[i][c][1] = 0.0;
    // 64 rows x 32 columns of x and of the router rows per chunk: 512 float4
    // each, two of each per thread
    float4 xv[2], wv[2];
    auto gload = [&](int kc) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = tid + 256 * u, r = i >> 3, k4 = i & 7;
            const int t = t0 + r, e = e0 + r;
            xv[u] = t < T ? __ldg(reinterpret_cast<const float4*>(x + (int64_t)t * H + kc * kRtK) + k4)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
            wv[u] = e < E ? __ldg(reinterpret_cast<const float4*>(Wr + (int64_t)e * H + kc * kRtK) + k4)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    if (kc0 < kc1) gload(kc0);
    for (int kc = kc0; kc < kc1; ++kc) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            // row r, columns 4 k4 .. 4 k4 + 3 as two 16-byte stores; lanes
            // with k4 >= 4 store their upper half first, so that each
            // store instruction of 8 lanes covers all 32 banks once
            const int i = tid + 256 * u, r = i >> 3, k4 = i & 7;
            const bool sw = k4 >= 4;
            double2* xr = reinterpret_cast<double2*>(&xs[r][4 * k4]);
            double2* wr = reinterpret_cast<double2*>(&ws[r][4 * k4]);
            const double2 xlo = make_double2((double)xv[u].x, (double)xv[u].y);
            const double2 xhi = make_double2((double)xv[u].z, (double)xv[u].w);
            const double2 wlo = make_double2((double)wv[u].x, (double)wv[u].y);
            const double2 whi = make_double2((double)wv[u].z, (double)wv[u].w);
            xr[sw ? 1 : 0] = sw ? xhi : xlo;
            wr[sw ? 1 : 0] = sw ? whi : wlo;
            xr[sw ? 0 : 1] = sw ? xlo : xhi;
            wr[sw ? 0 : 1] = sw ? wlo : whi;
        }
        __syncthreads();
        if (kc + 1 < kc1) gload(kc + 1);
#pragma unroll
        for (int k0 = 0; k0 < kRtK; k0 += 4) {
            double a[4], b[2];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = xs[wt + 8 * i + g][k0 + q];
#pragma unroll
            for (int c = 0; c < 2; ++c) b[c] = ws[we + 8 * c + g][k0 + q];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int c = 0; c < 2; ++c) dmma_8x8x4(acc[i][c], a[i], b[c]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + wt + 8 * i + g;
        if (t >= T) continue;
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int e = e0 + we + 8 * c + 2 * q + j;
                if (e < E) parts[((int64_t)split * T + t) * E + e] = acc[i][c][j];
            }
    }
}

__global__ void __launch_bounds__(256) k_router_reduce(const double* __restrict__ parts, int S, int64_t n,
                                                       double* __restrict__ logits) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        double v = parts[i];
        int sp = 1;
        // eight loads in flight at a time; the adds stay in split order
        for (; sp + 8 <= S; sp += 8) {
            double u[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) u[j] = parts[(int64_t)(sp + j) * n + i];
#pragma unroll
            for (int j = 0; j < 8; ++j) v = __dadd_rn(v, u[j]);
        }
        for (; sp < S; ++sp) v = __dadd_rn(v, parts[(int64_t)sp * n + i]);
        logits[i] = v;
    }
}

// Selection: one warp per token.  s = sigmoid(logit), c = s + bias; group
// score = sum of the two largest c (first the maximum, then the largest of the
// rest, ties to the lower index); keep the topk_groups best groups; take the
// top_k largest c in them, best first; w = s / sum(s) * rsf.  With topp in
// (0, 1) the adaptive expert top-p then drops the picks past the share
// prefix that reaches topp (idx -1, w 0) and renormalises the rest.
__global__ void __launch_bounds__(128) k_router_select(const double* __restrict__ logits,
                                                       const float* __restrict__ bias, int T, int E, int G,
                                                       int tg, int k, float rsf, float topp,
                                                       int32_t* __restrict__ idx, float* __restrict__ wout) {
    extern __shared__ double sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 4 + warp;
    double* sc = sm + (size_t)warp * 2 * E;  // c[E] then s[E]
    double* ss = sc + E;
    if (t >= T) return;
    const int per = E / G;
    for (int e = lane; e < E; e += 32) {
        const double l = logits[(int64_t)t * E + e];
        const double s = 1.0 / (1.0 + exp(-l));
        ss[e] = s;
        sc[e] = s + (double)bias[e];
    }
    __syncwarp();
    // group scores, one lane per group
    double gs = -INFINITY;
    if (lane < G) {
        int a = -1, b = -1;
        for (int e = lane * per; e < (lane + 1) * per; ++e)
            if (a < 0 || sc[e] > sc[a]) a = e;
        for (int e = lane * per; e < (lane + 1) * per; ++e)
            if (e != a && (b < 0 || sc[e] > sc[b])) b = e;
        gs = sc[a] + sc[b];
    }
    // keep tg groups
    uint32_t kept = 0;
    for (int n = 0; n < tg; ++n) {
        double v = (lane < G && !((kept >> lane) & 1u)) ? gs : -INFINITY;
        int i = (lane < G && !((kept >> lane) & 1u)) ? lane : 0x7fffffff;
        warp_argmax(v, i);
        if (i >= G) i = 0;  // only reachable with non-finite scores; keeps the shift defined
        kept |= 1u << i;
    }
    // top_k experts of the kept groups
    int sel_mine = -1;  // lane j < k holds the j-th pick
    double ssum = 0.0;
    for (int n = 0; n < k; ++n) {
        double v = -INFINITY;
        int i = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {
            if (!((kept >> (e / per)) & 1u)) continue;
            const double c = sc[e];
            if (c > v || (c == v && e < i)) {
                v = c;
                i = e;
            }
        }
        warp_argmax(v, i);
        if (i >= E) i = 0;  // only reachable with non-finite scores; keeps the access in bounds
        if (lane == (i & 31)) sc[i] = -INFINITY;  // owner lane marks it taken
        __syncwarp();
        if (lane == n) sel_mine = i;
        ssum += ss[i];  // same order as the picks: s_0 + s_1 + ...
    }
    if (topp > 0.f && topp < 1.f) {
        const double sj = lane < k ? ss[sel_mine] : 0.0;
        double skept;
        const bool keep = topp_keep(sj, ssum, k, topp, lane, &skept);
        if (lane < k) {
            idx[(int64_t)t * k + lane] = keep ? sel_mine : -1;
            wout[(int64_t)t * k + lane] = keep ? (float)(sj / skept * (double)rsf) : 0.f;
        }
        return;
    }
    if (lane < k) {
        idx[(int64_t)t * k + lane] = sel_mine;
        wout[(int64_t)t * k + lane] = (float)(ss[sel_mine] / ssum * (double)rsf);
    }
}

// The same selection for groups of 32 experts (warp g = group g), one CTA
// per token and one thread per expert, by ranks instead of rounds: a group
// is kept when fewer than topk_groups groups beat its score (larger, ties to
// the lower group), an expert of a kept group is pick r when r experts of
// the kept groups beat it (larger c, ties to the lower index) -- the order
// in which the rounds of k_router_select take them, so the picks, their
// order and the weights are the same.
__global__ void __launch_bounds__(1024) k_router_select_g32(const double* __restrict__ logits,
                                                            const float* __restrict__ bias, int E, int G, int tg,
                                                            int k, float rsf, float topp, int32_t* __restrict__ idx,
                                                            float* __restrict__ wout) {
    __shared__ double sc[1024], ss[1024], gsc[32];
    __shared__ int kg[32], sel[32];
    const int t = blockIdx.x, e = threadIdx.x, warp = e >> 5, lane = e & 31;
    if (e < 32) {  // in bounds whatever the scores (non-finite ones rank nothing)
        kg[e] = 0;
        sel[e] = 0;
    }
    {
        const double l = logits[(int64_t)t * E + e];
        const double sv = 1.0 / (1.0 + exp(-l));
        ss[e] = sv;
        sc[e] = sv + (double)bias[e];
    }
    __syncwarp();
    // group score: the sum of the group's two best c (ties to the lower index)
    {
        const double c = sc[e];
        double v = c;
        int a = e;
        warp_argmax(v, a);
        double v2 = e == a ? -INFINITY : c;
        int b = e == a ? 0x7fffffff : e;
        warp_argmax(v2, b);
        if (lane == 0) gsc[warp] = sc[a] + sc[b & 1023];
    }
    __syncthreads();
    if (e < G) {
        const double gs = gsc[e];
        int rank = 0;
        for (int g2 = 0; g2 < G; ++g2) rank += (gsc[g2] > gs || (gsc[g2] == gs && g2 < e)) ? 1 : 0;
        if (rank < tg) kg[rank] = e;
    }
    __syncthreads();
    // rank of this expert among the kept groups' experts
    bool mine = false;
    for (int q = 0; q < tg; ++q) mine |= kg[q] == warp;
    if (mine) {
        const double c = sc[e];
        int rank = 0;
        for (int q = 0; q < tg; ++q) {
            const int g2 = kg[q];
#pragma unroll 8
            for (int l2 = 0; l2 < 32; ++l2) {
                const int e2 = 32 * g2 + l2;
                const double c2 = sc[e2];
                rank += (c2 > c || (c2 == c && e2 < e)) ? 1 : 0;
            }
        }
        if (rank < k) sel[rank] = e;
    }
    __syncthreads();
    if (warp != 0) return;
    const int pick = lane < k ? sel[lane] : 0;
    const double sj = lane < k ? ss[pick] : 0.0;
    double ssum = 0.0;
    for (int n = 0; n < k; ++n) ssum += __shfl_sync(kFull, sj, n);  // pick order: s_0 + s_1 + ...
    if (topp > 0.f && topp < 1.f) {
        double skept;
        const bool keep = topp_keep(sj, ssum, k, topp, lane, &skept);
        if (lane < k) {
            idx[(int64_t)t * k + lane] = keep ? pick : -1;
            wout[(int64_t)t * k + lane] = keep ? (float)(sj / skept * (double)rsf) : 0.f;
        }
        return;
    }
    if (lane < k) {
        idx[(int64_t)t * k + lane] = pick;
        wout[(int64_t)t * k + lane] = (float)(sj / ssum * (double)rsf);
    }
}

size_t router_ws_bytes(const moe_config& c, int T) {
    const size_t logits = ((size_t)T * c.n_experts * sizeof(double) + 255) & ~(size_t)255;
    const int S = router_splits(c, T);
    return logits + (size_t)S * T * c.n_experts * sizeof(double);
}

cudaError_t launch_router(const moe_config& c, const float* x, int T, const float* router_w,
                          const float* bias, double* logits, int32_t* idx, float* w, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    cudaError_t e;
    const int S = router_splits(c, T);
    if (S > 0) {
        // the partial sums follow the logits in the router's workspace
        double* parts = logits + (((size_t)T * c.n_experts * sizeof(double) + 255) & ~(size_t)255) / sizeof(double);
        const int chunks = c.hidden / kRtK;
        const int per = (chunks + S - 1) / S;
        dim3 g0((c.n_experts + kRtE - 1) / kRtE, (T + kRtT - 1) / kRtT, S);
        k_router_logits_f64<<<g0, 256, 0, s>>>(x, T, c.hidden, router_w, c.n_experts, per, parts);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        const int64_t n = (int64_t)T * c.n_experts;
        const int64_t want = (n + 255) / 256, cap = (int64_t)device_info().sm_count * 8;
        k_router_reduce<<<(int)(want < cap ? want : cap), 256, 0, s>>>(parts, S, n, logits);
    } else {
        dim3 g1((c.n_experts + kRouterExpertsPerCta - 1) / kRouterExpertsPerCta,
                (T + kRouterTokens - 1) / kRouterTokens);
        k_router_logits<<<g1, 256, 0, s>>>(x, T, c.hidden, router_w, c.n_experts, logits);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (c.n_experts / c.n_groups == 32 && c.top_k <= 32) {  // E = 32 G <= 1024: one thread per expert
        k_router_select_g32<<<T, c.n_experts, 0, s>>>(logits, bias, c.n_experts, c.n_groups, c.topk_groups,
                                                      c.top_k, c.routed_scaling_factor, c.expert_topp, idx, w);
        return cudaGetLastError();
    }
    const size_t smem = (size_t)4 * 2 * c.n_experts * sizeof(double);
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(k_router_select, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_router_select<<<(T + 3) / 4, 128, smem, s>>>(logits, bias, T, c.n_experts, c.n_groups, c.topk_groups,
                                                   c.top_k, c.routed_scaling_factor, c.expert_topp, idx, w);
    return cudaGetLastError();
}

}  // namespace moe
