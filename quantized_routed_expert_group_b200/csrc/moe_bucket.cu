// moe_bucket.cu -- batch-union bucketing of (token, slot) pairs by expert.
//
// GeekNews "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", §구현된 주요 기능 ("Batch-union
// MoE": each unique expert of a prefill / MTP-verify batch is read once and
// applied to every position routed to it); wpnews.pro "Colibri — รัน GLM-5.2
// ...", "Batch-Union MoE".  The bucket order is a stable counting sort: within
// an expert, pairs keep increasing token order.  A token never picks the same
// expert twice, so the rank of (t, j) inside bucket e is the number of earlier
// tokens that picked e: one bit per (expert, token) and a popcount give it
// without atomics on the order.  A pair the adaptive top-p dropped (idx -1)
// is in no bucket: it gets inv_perm -1, and perm ends with -1 for each.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kBucketThreads = 1024;

size_t bucket_smem_bytes(const moe_config& c, int T) {
    const size_t words = (size_t)c.n_experts * (size_t)((T + 31) / 32);
    return words * 4 + (size_t)(c.n_experts + 1) * 4 * 2 + 64 * 4;
}

// Exclusive scan of in[0..n) (n <= 1024) by a 1024-thread CTA; returns the
// total.  scratch: 32 ints.
__device__ int cta_exclusive_scan(const int* in, int* out, int n, int* scratch) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int v = tid < n ? in[tid] : 0;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += u;
    }
    if (lane == 31) scratch[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int s = scratch[lane];
        int si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(kFull, si, o);
            if (lane >= o) si += u;
        }
        scratch[lane] = si - s;  // exclusive prefix of warp totals
        if (lane == 31) scratch[32] = si;
    }
    __syncthreads();
    if (tid < n) out[tid] = inc - v + scratch[warp];
    const int total = scratch[32];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(kBucketThreads) k_bucket(const int32_t* __restrict__ idx, int T, int k, int E,
                                                           int32_t* __restrict__ counts,
                                                           int32_t* __restrict__ offsets,
                                                           int32_t* __restrict__ perm,
                                                           int32_t* __restrict__ inv_perm,
                                                           int32_t* __restrict__ active, int32_t* err) {
    extern __shared__ uint32_t smem[];
    const int W = (T + 31) / 32;
    uint32_t* mask = smem;                                     // [E][W]
    int* cnt = reinterpret_cast<int*>(mask + (size_t)E * W);   // [E+1]
    int* off = cnt + (E + 1);                                  // [E+1]
    int* scratch = off + (E + 1);                              // [64]
    const int tid = threadIdx.x;
    const int n = T * k;
    for (int i = tid; i < E * W; i += kBucketThreads) mask[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kBucketThreads) {
        const int e = idx[i];
        if (e < 0 || e >= E) {
            if (e != -1) set_error(err, kErrIndex);
            continue;
        }
        const int t = i / k;
        atomicOr(&mask[(size_t)e * W + (t >> 5)], 1u << (t & 31));
    }
    __syncthreads();
    for (int e = tid; e < E; e += kBucketThreads) {
        int c = 0;
        for (int w = 0; w < W; ++w) c += __popc(mask[(size_t)e * W + w]);
        cnt[e] = c;
    }
    __syncthreads();
    const int total = cta_exclusive_scan(cnt, off, E, scratch);
    if (tid == 0) off[E] = total;
    __syncthreads();
    for (int e = tid; e <= E; e += kBucketThreads) {
        offsets[e] = off[e];
        if (e < E) counts[e] = cnt[e];
    }
    for (int i = tid; i < n; i += kBucketThreads) {
        const int e = idx[i];
        if (e < 0 || e >= E) {
            if (inv_perm) inv_perm[i] = -1;
            continue;
        }
        const int t = i / k;
        const uint32_t* m = mask + (size_t)e * W;
        int r = __popc(m[t >> 5] & ((1u << (t & 31)) - 1u));
        for (int w = 0; w < (t >> 5); ++w) r += __popc(m[w]);
        const int p = off[e] + r;
        perm[p] = i;
        if (inv_perm) inv_perm[i] = p;
    }
    for (int i = total + tid; i < n; i += kBucketThreads) perm[i] = -1;  // dropped pairs
    // active experts (count > 0) in increasing id order
    if (!active) return;  // uniform across the CTA
    __syncthreads();
    for (int e = tid; e < E; e += kBucketThreads) cnt[e] = cnt[e] > 0 ? 1 : 0;
    __syncthreads();
    const int n_act = cta_exclusive_scan(cnt, off, E, scratch);
    for (int e = tid; e < E; e += kBucketThreads)
        if (cnt[e]) active[1 + off[e]] = e;
    if (tid == 0) active[0] = n_act;
}

cudaError_t launch_bucket(const moe_config& c, const int32_t* idx, int T, int32_t* counts, int32_t* offsets,
                          int32_t* perm, int32_t* inv_perm, int32_t* active, int32_t* err, cudaStream_t s) {
    const size_t smem = bucket_smem_bytes(c, T);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_bucket, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_bucket<<<1, kBucketThreads, smem, s>>>(idx, T, c.top_k, c.n_experts, counts, offsets, perm, inv_perm,
                                              active, err);
    return cudaGetLastError();
}

__global__ void k_ep_mask(const int32_t* __restrict__ idx, int64_t n, int lo, int hi, int32_t* __restrict__ out) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int e = idx[i];
        out[i] = (e >= lo && e < hi) ? e : -1;
    }
}

cudaError_t launch_ep_mask(const int32_t* idx, int64_t n, int lo, int hi, int32_t* idx_ep, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const int64_t want = (n + 255) / 256;
    k_ep_mask<<<(int)(want < 1024 ? want : 1024), 256, 0, s>>>(idx, n, lo, hi, idx_ep);
    return cudaGetLastError();
}

}  // namespace moe
