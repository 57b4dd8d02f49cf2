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

cudaError_t launch_router(const moe_config& c, const float* x, int T, const float* router_w,
                          const float* bias, double* logits, int32_t* idx, float* w, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    dim3 g1((c.n_experts + kRouterExpertsPerCta - 1) / kRouterExpertsPerCta,
            (T + kRouterTokens - 1) / kRouterTokens);
    k_router_logits<<<g1, 256, 0, s>>>(x, T, c.hidden, router_w, c.n_experts, logits);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
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
