// moe_tc.cu -- the batched expert path on tcgen05 tensor cores (sm_100a) and
// its host-side plumbing (tensor maps).
//
// GeekNews "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", §구현된 주요 기능: the expert
// matmuls multiply Q8_0-style int8 activations (one fp32 scale per 32 values)
// by packed int4 / int8 weights with per-row scales; "Batch-union MoE" applies
// each unique expert once to every position routed to it.  wpnews.pro
// "Colibri — รัน GLM-5.2 ...", kernel table (int4 packed, dequant-on-use; the
// int4 path is faster "in batch").  With hundreds of tokens a batch-union
// expert meets tens to hundreds of tokens per weight row, so the contraction
// is dense enough for the tensor cores: one kind::i8 MMA (K = 32 = one Q8_0
// block) per block gives the exact int32 block dots of a 128-row weight tile
// with up to 64 tokens, and the per-token block scales are applied to them
// from TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_device.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"
#include "moe_tc.cuh"

namespace moe {
namespace tc {

// ---------------------------------------------------------------------------
// Tensor maps (host)
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D map of a row-major array [rows][cols] of elements of type dtype with box
// [box_rows][box_cols]; out-of-range elements of a box read as zero.
cudaError_t encode_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t cols, uint64_t rows,
                      uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
    const PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, dtype, 2,
                          const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Staging box of one stage of packed weight rows: the swizzle that makes the
// widening reads conflict-free (int8 rows go straight into the MMA layout).
template <int WBITS>
constexpr CUtensorMapSwizzle raw_swizzle() {
    return WBITS == 8 ? CU_TENSOR_MAP_SWIZZLE_128B : WBITS == 4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
}

cudaError_t encode_weights(CUtensorMap* map, const uint8_t* w, int64_t rows, int cols, int wbits) {
    const uint64_t rb = (uint64_t)cols * wbits / 8;
    const CUtensorMapSwizzle swz = wbits == 8 ? raw_swizzle<8>() : wbits == 4 ? raw_swizzle<4>() : raw_swizzle<2>();
    return encode_2d(map, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, rb, (uint64_t)rows, rb, (uint32_t)(kStageK * wbits / 8),
                     kTileRows, swz);
}

// ---------------------------------------------------------------------------
// Per-block dot export through the tensor-core routine
// ---------------------------------------------------------------------------
// One CTA per 128-row weight tile, four warps, a synchronous loop over the
// stages: TMA of the packed rows and of the token codes, widening into the
// MMA layout, one kind::i8 MMA per Q8_0 block into its own TMEM accumulator,
// and the raw int32 dots read back from TMEM.
struct DotsSmem {
    static constexpr int kA = 0;                                // widened weight tile, 16 KB
    static constexpr int kX = kA + kTileBytes;                  // token codes, 64 x 128 B
    static constexpr int kRaw = kX + kMaxN * kStageK;           // packed staging, <= 8 KB
    static constexpr int kBar = kRaw + kTileRows * kStageK / 2; // barriers, TMEM address
    static constexpr int kBytes = kBar + 64;
};
constexpr int kDotsThreads = 128;
constexpr uint64_t kExportWaitNs = 100ull * 1000 * 1000;
// + alignment slack; at least 120 KB so that one CTA runs per SM and its TMEM
// allocation never waits for another CTA's
constexpr int kDotsSmem = DotsSmem::kBytes + 1024 > 120 * 1024 ? DotsSmem::kBytes + 1024 : 120 * 1024;

template <int WBITS>
__global__ void __launch_bounds__(kDotsThreads) k_tc_block_dots(const __grid_constant__ CUtensorMap wmap,
                                                                const __grid_constant__ CUtensorMap qmap,
                                                                int64_t rows, int cols, int n,
                                                                int32_t* __restrict__ out) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* a_tile = sm + DotsSmem::kA;
    uint8_t* x_tile = sm + DotsSmem::kX;
    uint8_t* raw = WBITS == 8 ? a_tile : sm + DotsSmem::kRaw;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + DotsSmem::kBar);
    uint64_t* done = full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t row0 = (int64_t)blockIdx.x * kTileRows;
    const int nb = cols / 32;
    const int nstage = (cols + kStageK - 1) / kStageK;
    const int N = (n + 15) & ~15;
    constexpr uint32_t kRawBytes = kTileRows * raw_row_bytes<WBITS>();
    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(done, 1);
        fence_barrier_init();
        tma_prefetch_map(&wmap);
        tma_prefetch_map(&qmap);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    for (int s = 0; s < nstage; ++s) {
        if (tid == 0) {
            mbar_arrive_expect_tx(full, kRawBytes + (uint32_t)(kMaxN * kStageK));
            tma_load_2d(raw, &wmap, s * raw_row_bytes<WBITS>(), (int)row0, full);
            tma_load_2d(x_tile, &qmap, s * kStageK, 0, full);
        }
        // a uniform decision: every thread leaves, or none
        if (__syncthreads_or(mbar_wait_ns(full, s & 1, kExportWaitNs) ? 0 : 1)) break;
        if constexpr (WBITS != 8) widen_row<WBITS>(raw, a_tile, tid);
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after_sync();
            const uint64_t ad = desc_k128_sw128(a_tile), bd = desc_k128_sw128(x_tile);
#pragma unroll
            for (int j = 0; j < kBlocksPerStage; ++j)
                mma_i8(tmem + (uint32_t)(j * kMaxN), ad + 2 * j, bd + 2 * j, idesc_i8(N), false);
            mma_commit(done);
        }
        if (__syncthreads_or(mbar_wait_ns(done, s & 1, kExportWaitNs) ? 0 : 1)) break;
        tc_fence_after_sync();
        const int64_t r = row0 + warp * 32 + lane;
#pragma unroll 1
        for (int j = 0; j < kBlocksPerStage; ++j) {
            const int b = s * kBlocksPerStage + j;
#pragma unroll 1
            for (int g = 0; g < N; g += 16) {
                uint32_t v[16];
                tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(j * kMaxN + g), v);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int t = g + c;
                    if (t < n && r < rows && b < nb) out[((int64_t)t * rows + r) * nb + b] = (int32_t)v[c];
                }
            }
        }
        tc_fence_before_sync();
        __syncthreads();
    }
    tc_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

}  // namespace tc

cudaError_t launch_tc_block_dots(const uint8_t* packed, int64_t rows, int cols, int wbits, const int8_t* q, int n,
                                 int32_t* out, cudaStream_t s) {
    using namespace tc;
    if (n > kMaxN || rows > (int64_t)0x7FFFFFFF) return cudaErrorInvalidValue;
    CUtensorMap wm, qm;
    cudaError_t e = encode_weights(&wm, packed, rows, cols, wbits);
    if (e != cudaSuccess) return e;
    e = encode_2d(&qm, q, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)cols, (uint64_t)n, (uint64_t)cols, kStageK, kMaxN,
                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((rows + kTileRows - 1) / kTileRows);
    auto run = [&](auto kernel) {
        cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDotsSmem);
        if (r != cudaSuccess) return r;
        kernel<<<grid, kDotsThreads, kDotsSmem, s>>>(wm, qm, rows, cols, n, out);
        return cudaGetLastError();
    };
    if (wbits == 4) return run(k_tc_block_dots<4>);
    if (wbits == 2) return run(k_tc_block_dots<2>);
    return run(k_tc_block_dots<8>);
}



// ===========================================================================
// The batched expert path: plan, gather, grouped GEMMs, SwiGLU
// ===========================================================================
//
// Data flow (T at or above kTcMinTokens, see tc_path_supported):
//   Q8_0 of x, router, bucketing   (the multi-kernel path's kernels)
//   k_tc_plan     the batch-union entries (each selected expert, then
//                 the shared expert), their rows in a padded row space (each
//                 entry's tokens start on a multiple of 16 rows), and the work
//                 units (entry, 128-row weight tile, matrix, chunk of <= 64
//                 tokens), heaviest entries first; every CTA of a few builds
//                 the entry tables, and they split the units and rows
//   k_tc_gather   the entries' Q8_0 codes of x into the padded row space
//                 (xg [prows][hidden]) and their block scales, transposed and
//                 widened to fp64 (xdT [hidden/32][prows]), so that every
//                 unit's tokens are one TMA box
//   k_tc_gemm     gate/up: g and u row values per padded row (gu [2][prows][inter])
//   k_tc_swiglu   h = silu(g) * u and Q8_0 of h -> hg / hdT (padded rows, for
//                 the down GEMM) and hq / hd (per slot)
//   k_tc_gemm     down: y per slot
//   k_combine     (the multi-kernel path's)
//
// Arithmetic: a row value is s_row * sum_b d_b * dot_b with the int32 block
// dots from the tensor core; the epilogue adds d_b * dot_b in fp64 in block
// order (each product is exact in fp64), multiplies by s_row in fp64 and
// rounds to fp32, and SwiGLU is evaluated in fp64 and rounded to fp32 before
// Q8_0 -- the same operations in the same order as the definition, so the h
// codes do not depend on a summation order.  (fp64 on the B200's CUDA cores
// runs at half the fp32 rate; a 32 x 32 -> 64-bit integer multiply-add, the
// alternative for exact sums, at a sixth.)
namespace tc {

struct PlanParams {
    int T, k, E, ns, I, H;
    int prows_cap;
    int units_gu_cap, units_dn_cap;
    const int32_t* offsets;
    const int32_t* perm;
    const int32_t* active;
    TcUnit* units_gu;
    TcUnit* units_dn;
    int32_t* row_tok;
    int32_t* row_slot;
    int32_t* ctrl;  // [0] gate/up units, [1] down units, [2] padded rows, [3] gate/up counter, [4] down counter
    int32_t* err;
};

constexpr int kPlanThreads = 1024;
constexpr int kPlanCtas = 16;  // every CTA builds the entry tables; the units and rows are split over them
constexpr int kMaxEntries = 1025;
constexpr int kUnitUp = 1 << 17;  // TcUnit::info: the unit's matrix is W_up (gate/up GEMM)

// Exclusive scan of one value per thread over the CTA (kPlanThreads threads,
// every thread calls it); returns the prefix and sets *total.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = warp_sums[lane];
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(kFull, wi, o);
            if (lane >= o) wi += u;
        }
        warp_sums[lane] = wi - w;  // exclusive over warps
        if (lane == 31) warp_sums[32] = wi;
    }
    __syncthreads();
    const int r = warp_sums[warp] + incl - v;
    *total = warp_sums[32];
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(kPlanThreads) k_tc_plan(PlanParams p) {
    __shared__ int s_n[kMaxEntries], s_slot0[kMaxEntries], s_prow0[kMaxEntries], s_sched[kMaxEntries];
    __shared__ int s_ugu0[kMaxEntries], s_udn0[kMaxEntries];
    __shared__ int s_ws[33];
    const int tid = threadIdx.x;
    const int umax = p.E < p.T * p.k ? p.E : p.T * p.k;
    int U = p.active[0];
    U = U < 0 ? 0 : (U > umax ? umax : U);
    const int ne = U + p.ns;
    const int tiles_gu = p.I / kTileRows, tiles_dn = p.H / kTileRows;
    for (int i = tid; i < ne; i += kPlanThreads) {
        if (i < U) {
            int e = p.active[1 + i];
            if (e < 0 || e >= p.E) {
                set_error(p.err, kErrIndex);
                e = 0;
            }
            s_slot0[i] = p.offsets[e];
            s_n[i] = p.offsets[e + 1] - p.offsets[e];
        } else {
            s_slot0[i] = p.T * p.k;
            s_n[i] = p.T;
        }
    }
    __syncthreads();
    // padded rows: each entry starts on a multiple of 16
    int run = 0;
    for (int base = 0; base < ne; base += kPlanThreads) {
        const int i = base + tid;
        const int v = i < ne ? (s_n[i] + 15) & ~15 : 0;
        int tot;
        const int ex = block_excl_scan(v, s_ws, &tot);
        if (i < ne) s_prow0[i] = run + ex;
        run += tot;
    }
    const int prows = run;
    // schedule: entries by decreasing token count (ties: lower entry first)
    for (int i = tid; i < ne; i += kPlanThreads) {
        const int ni = s_n[i];
        int rank = 0;
        for (int j = 0; j < ne; ++j) rank += (s_n[j] > ni || (s_n[j] == ni && j < i)) ? 1 : 0;
        s_sched[rank] = i;
    }
    __syncthreads();
    int rgu = 0, rdn = 0;
    for (int base = 0; base < ne; base += kPlanThreads) {
        const int r = base + tid;
        const int nch = r < ne ? (s_n[s_sched[r]] + kChunk - 1) / kChunk : 0;
        int tg, td;
        const int eg = block_excl_scan(2 * nch * tiles_gu, s_ws, &tg);
        const int ed = block_excl_scan(nch * tiles_dn, s_ws, &td);
        if (r < ne) {
            s_ugu0[r] = rgu + eg;
            s_udn0[r] = rdn + ed;
        }
        rgu += tg;
        rdn += td;
    }
    if (prows > p.prows_cap || rgu > p.units_gu_cap || rdn > p.units_dn_cap) {
        // cannot happen for a consistent bucketing; leave no work
        if (blockIdx.x == 0 && tid == 0) {
            set_error(p.err, kErrIndex);
            for (int i = 0; i < 5; ++i) p.ctrl[i] = 0;
        }
        return;
    }
    // work units: per entry (in schedule order) by weight tile, then matrix,
    // then token chunk, so that the chunks of one weight tile follow each
    // other; every thread writes units, each finding its entry by a binary
    // search over the entries' first unit
    auto entry_of = [&](const int* first, int u) {
        int lo = 0, hi = ne - 1;
        while (lo < hi) {  // last entry (schedule rank) whose first unit is <= u
            const int mid = (lo + hi + 1) >> 1;
            if (first[mid] <= u) lo = mid;
            else hi = mid - 1;
        }
        return lo;
    };
    const int g0 = blockIdx.x * kPlanThreads + tid, gstep = gridDim.x * kPlanThreads;
    for (int u = g0; u < rgu; u += gstep) {
        const int r = entry_of(s_ugu0, u), i = s_sched[r];
        const int n = s_n[i], nch = (n + kChunk - 1) / kChunk;
        const int l = u - s_ugu0[r], c = l % nch, tm = l / nch, m = tm & 1, t = tm >> 1;
        const bool shared = i >= U;
        TcUnit w;
        w.prow0 = s_prow0[i] + c * kChunk;
        w.ntok = min(kChunk, n - c * kChunk);
        w.wrow0 = (shared ? 0 : p.active[1 + i]) * p.I + t * kTileRows;
        w.info = t | (shared ? kUnitShared : 0) | (m ? kUnitUp : 0);
        p.units_gu[u] = w;
    }
    for (int u = g0; u < rdn; u += gstep) {
        const int r = entry_of(s_udn0, u), i = s_sched[r];
        const int n = s_n[i], nch = (n + kChunk - 1) / kChunk;
        const int l = u - s_udn0[r], c = l % nch, t = l / nch;
        const bool shared = i >= U;
        TcUnit w;
        w.prow0 = s_prow0[i] + c * kChunk;
        w.ntok = min(kChunk, n - c * kChunk);
        w.wrow0 = (shared ? 0 : p.active[1 + i]) * p.H + t * kTileRows;
        w.info = t | (shared ? kUnitShared : 0);
        p.units_dn[u] = w;
    }
    // padded row -> token and slot (-1 for the padding rows)
    for (int q = g0; q < prows; q += gstep) {
        int lo = 0, hi = ne - 1;
        while (lo < hi) {  // last entry whose first row is <= q
            const int mid = (lo + hi + 1) >> 1;
            if (s_prow0[mid] <= q) lo = mid;
            else hi = mid - 1;
        }
        const int j = q - s_prow0[lo];
        int tok = -1, slot = -1;
        if (j < s_n[lo]) {
            slot = s_slot0[lo] + j;
            tok = lo < U ? p.perm[slot] / p.k : j;
        }
        p.row_tok[q] = tok;
        p.row_slot[q] = slot;
    }
    if (blockIdx.x == 0 && tid == 0) {
        p.ctrl[0] = rgu;
        p.ctrl[1] = rdn;
        p.ctrl[2] = prows;
        p.ctrl[3] = 0;
        p.ctrl[4] = 0;
    }
}

// Q8_0 of x, one CTA per token (as k_quantize_q8_0: one warp per block of 32,
// lane = element), and the token's digit planes [5][hidden] with its 2^E
// (see kPlanes).  A token whose block-scale exponents spread over more than
// kMaxSpread sets *wide; the call then takes the fp64-epilogue GEMMs and the
// planes are not used.
constexpr int kQuantThreads = 256;
constexpr int kMaxQuantCols = 8192;  // hidden and inter of the batched path

// Row quantisers of the batched path, four consecutive elements a thread:
// a Q8_0 block of 32 is eight lanes, and a thread keeps its codes in
// registers between the row's two passes (Q8_0, then the digit planes,
// which need the smallest block exponent E of the whole row).
constexpr int kQuadSpan = 4 * kQuantThreads;           // elements of a row per pass of the CTA
constexpr int kQuadIters = kMaxQuantCols / kQuadSpan;  // passes at the widest row

// Q8_0 of four values of a block whose other 28 sit in the thread's seven
// neighbours (lanes 8j .. 8j+7): the arithmetic of q8_0_warp (d = amax/127,
// q = round-half-away(v * (1/d)) clamped to [-127, 127], amax < FLT_MIN gives
// d = 0 and zero codes); returns the four codes packed, element 0 lowest.
// Every lane of the warp must call it.
__device__ __forceinline__ uint32_t q8_0_quad(const float (&v)[4], float& d) {
    float a = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
    d = 0.0f;
    if (!(a >= FLT_MIN)) return 0u;
    d = __fdiv_rn(a, 127.0f);
    const float id = __fdiv_rn(1.0f, d);
    uint32_t b4[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) b4[e] = (uint32_t)(int)fminf(fmaxf(roundf(__fmul_rn(v[e], id)), -127.0f), 127.0f);
    return __byte_perm(__byte_perm(b4[0], b4[1], 0x0040), __byte_perm(b4[2], b4[3], 0x0040), 0x5410);
}

// The row's smallest and largest block exponent over its nonzero blocks (the
// mantissas and exponents of its nb block scales in shared memory), the
// same in every thread (emin > emax: all blocks zero).  Every thread of the
// CTA calls it, after the scales are written and a __syncthreads.
__device__ __forceinline__ void row_exp_span(const uint32_t* s_m, const int* s_e, int nb, int* s_red, int& emin,
                                             int& emax) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    emin = 0x7FFFFFFF;
    emax = -0x7FFFFFFF;
    for (int b = threadIdx.x; b < nb; b += blockDim.x)
        if (s_m[b]) {
            emin = min(emin, s_e[b]);
            emax = max(emax, s_e[b]);
        }
    emin = __reduce_min_sync(kFull, emin);
    emax = __reduce_max_sync(kFull, emax);
    if (lane == 0) {
        s_red[warp] = emin;
        s_red[nw + warp] = emax;
    }
    __syncthreads();
    for (int w = 0; w < nw; ++w) {
        emin = min(emin, s_red[w]);
        emax = max(emax, s_red[nw + w]);
    }
}

// The kPlanes digit-plane words of four packed codes q_e (element 0 lowest)
// of one block with mantissa m (< 2^32): q m + 0x8080808080 lies in
// [0, 2^40) for |q| <= 127, and its bytes are the signed base-256 digits c_p
// of q m (q m = sum_p 256^p c_p, c_p in [-128, 127]) plus 128, so each plane
// word is a byte transpose of the four sums with the top bits flipped.
__device__ __forceinline__ void quad_planes(uint32_t codes, uint32_t m, uint32_t (&pw)[kPlanes]) {
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int qe = (int)(int8_t)(codes >> (8 * e));
        const uint64_t t = (uint64_t)((int64_t)qe * (int64_t)m) + 0x8080808080ull;
        lo[e] = (uint32_t)t;
        hi[e] = (uint32_t)(t >> 32);
    }
    const uint32_t a01 = __byte_perm(lo[0], lo[1], 0x5140), b01 = __byte_perm(lo[0], lo[1], 0x7362);
    const uint32_t a23 = __byte_perm(lo[2], lo[3], 0x5140), b23 = __byte_perm(lo[2], lo[3], 0x7362);
    pw[0] = __byte_perm(a01, a23, 0x5410) ^ 0x80808080u;
    pw[1] = __byte_perm(a01, a23, 0x7632) ^ 0x80808080u;
    pw[2] = __byte_perm(b01, b23, 0x5410) ^ 0x80808080u;
    pw[3] = __byte_perm(b01, b23, 0x7632) ^ 0x80808080u;
    pw[4] = __byte_perm(__byte_perm(hi[0], hi[1], 0x0040), __byte_perm(hi[2], hi[3], 0x0040), 0x5410) ^ 0x80808080u;
}

// Second pass of a row quantiser: the row's digit planes [kPlanes][n] from
// the codes the thread kept (codes[j]: the four elements from 4 (threadIdx.x
// + j kQuantThreads)) and 2^E to *pe (0 for an all-zero row); a row whose
// exponents spread over more than kMaxSpread sets *wide and writes no
// planes.  Every thread of the CTA calls it, after writing its block scales.
__device__ __forceinline__ void row_planes_quad(const uint32_t (&codes)[kQuadIters], const uint32_t* s_m,
                                                const int* s_e, int n, int* s_red, int8_t* __restrict__ planes,
                                                double* __restrict__ pe, int* wide) {
    __syncthreads();
    int emin, emax;
    row_exp_span(s_m, s_e, n / 32, s_red, emin, emax);
    const bool any = emin <= emax;  // some block is not zero
    if (any && emax - emin > kMaxSpread) {
        if (threadIdx.x == 0) atomicOr(wide, 1);
        return;
    }
#pragma unroll
    for (int j = 0; j < kQuadIters; ++j) {
        const int i = 4 * (threadIdx.x + j * kQuantThreads);
        if (i >= n) break;
        const int b = i >> 5;
        const uint32_t m = s_m[b] ? s_m[b] << (s_e[b] - emin) : 0u;
        uint32_t pw[kPlanes];
        quad_planes(codes[j], m, pw);
#pragma unroll
        for (int pl = 0; pl < kPlanes; ++pl) *reinterpret_cast<uint32_t*>(planes + (int64_t)pl * n + i) = pw[pl];
    }
    if (threadIdx.x == 0) *pe = any ? ldexp(1.0, emin) : 0.0;
}

// Q8_0 of x, one CTA per token (the arithmetic of k_quantize_q8_0, four
// elements a thread), and the token's digit planes [5][hidden] with its 2^E
// (see kPlanes); a token too wide for the planes sets *wide (the call then
// takes the fp64-epilogue GEMMs).  hidden is a multiple of 128, so a warp's
// 128 elements are all in the row or all past it.
__global__ void __launch_bounds__(kQuantThreads) k_tc_quantize(const float* __restrict__ x, int H,
                                                               int8_t* __restrict__ xq, float* __restrict__ xd,
                                                               int8_t* __restrict__ xpt, double* __restrict__ pet,
                                                               int* wide) {
    __shared__ uint32_t s_m[kMaxQuantCols / 32];
    __shared__ int s_e[kMaxQuantCols / 32];
    __shared__ int s_red[2 * kQuantThreads / 32];
    const int t = blockIdx.x, lane = threadIdx.x & 31;
    const int nb = H / 32;
    const float4* xt = reinterpret_cast<const float4*>(x + (int64_t)t * H);
    uint32_t codes[kQuadIters];
    float4 v = 4 * threadIdx.x < H ? __ldg(xt + threadIdx.x) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kQuadIters; ++j) {
        const int u = threadIdx.x + j * kQuantThreads, i = 4 * u;
        if (i >= H) break;
        // the next pass's load in flight
        const float4 vn = i + kQuadSpan < H ? __ldg(xt + u + kQuantThreads) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float vv[4] = {v.x, v.y, v.z, v.w};
        float d;
        codes[j] = q8_0_quad(vv, d);
        *reinterpret_cast<uint32_t*>(xq + (int64_t)t * H + i) = codes[j];
        if ((lane & 7) == 0) {
            const int b = i >> 5;
            xd[(int64_t)t * nb + b] = d;
            f32_mant_exp(d, s_m[b], s_e[b]);
        }
        v = vn;
    }
    row_planes_quad(codes, s_m, s_e, H, s_red, xpt + (int64_t)t * kPlanes * H, pet + t, wide);
}

// One warp per padded row: its token's digit planes and 2^E (zeros for a
// padding row); when some token is wide instead the token's Q8_0 codes and
// its block scales, transposed, as fp64 (for the fp64-epilogue GEMM).
__global__ void __launch_bounds__(256) k_tc_gather(const int8_t* __restrict__ xq, const float* __restrict__ xd,
                                                   const int8_t* __restrict__ xpt, const double* __restrict__ pet,
                                                   const int* __restrict__ wide, int H, int prows_cap,
                                                   const int32_t* __restrict__ row_tok,
                                                   const int32_t* __restrict__ ctrl, int8_t* __restrict__ xg,
                                                   double* __restrict__ xdT, int8_t* __restrict__ xp,
                                                   double* __restrict__ pex) {
    const int lane = threadIdx.x & 31;
    const int q = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (q >= ctrl[2]) return;
    const int tok = row_tok[q];
    if (!*wide) {
        const int n16 = kPlanes * H / 16;
        uint4* dst = reinterpret_cast<uint4*>(xp + (int64_t)q * kPlanes * H);
        const uint4* src = reinterpret_cast<const uint4*>(xpt + (int64_t)(tok < 0 ? 0 : tok) * kPlanes * H);
#pragma unroll 4
        for (int i = lane; i < n16; i += 32) dst[i] = tok >= 0 ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
        if (lane == 0) pex[q] = tok >= 0 ? pet[tok] : 0.0;
        return;
    }
    const int n16 = H / 16, nb = H / 32;
    uint4* dst = reinterpret_cast<uint4*>(xg + (int64_t)q * H);
    const uint4* src = reinterpret_cast<const uint4*>(xq + (int64_t)(tok < 0 ? 0 : tok) * H);
    for (int i = lane; i < n16; i += 32) dst[i] = tok >= 0 ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    for (int b = lane; b < nb; b += 32)
        xdT[(int64_t)b * prows_cap + q] = tok >= 0 ? (double)__ldg(xd + (int64_t)tok * nb + b) : 0.0;
}

// ---------------------------------------------------------------------------
// Grouped GEMM kernel (persistent, one CTA per SM, warp-specialised)
// ---------------------------------------------------------------------------
// warps 0-15  epilogue: warp w reads TMEM lanes 32 (w % 4) .. (its 32 weight
//             rows) and columns 16 (w / 4) .. (its 16 tokens); per Q8_0 block
//             it converts the int32 dots exactly to fp64 and accumulates
//             d_token * dot in fp64; at a unit's end it applies the row scale
//             (fp64, rounded to fp32) and writes g / u (gate/up) or y (down)
// warps 16-17 widening: packed int4 / int2 staging rows -> int8 MMA tiles
// warp 18     producer: takes units from a global counter, TMA of the packed
//             weight rows, the token codes and their block scales per stage
// warp 19     MMA: allocates TMEM; per block one kind::i8 MMA into one of
//             kNAcc accumulators, committed to the epilogue
// Every wait is bounded by the global timer and records kErrTimeout.
constexpr int kEpiWarps = 16;
constexpr int kConvWarps = 2;
constexpr int kProdWarp = kEpiWarps + kConvWarps;
constexpr int kMmaWarp = kProdWarp + 1;
constexpr int kGemmThreads = (kMmaWarp + 1) * 32;
constexpr int kNAcc = 8;
constexpr uint64_t kGemmWaitNs = 100ull * 1000 * 1000;

template <int WBITS>
struct GemmSmem {
    static constexpr int kRawTile = WBITS == 8 ? 0 : kTileRows * raw_row_bytes<WBITS>();
    static constexpr int kA = 0;                       // widened tile (int8: the TMA target)
    static constexpr int kX = kTileBytes;              // token codes [64][128]
    static constexpr int kRaw = kX + kMaxN * kStageK;  // packed staging tile
    static constexpr int kD = kRaw + kRawTile;         // block scales [4][64] fp64
    static constexpr int kStageBytes = (kD + kBlocksPerStage * kMaxN * 8 + 1023) & ~1023;
    static constexpr int kCtrl = 1024;
    static constexpr int kStagesFit = (220 * 1024 - kCtrl - 1024) / kStageBytes;
    static constexpr int kStages = kStagesFit < 6 ? kStagesFit : 6;
    static constexpr int kBytes = kStages * kStageBytes + kCtrl + 1024;  // + alignment slack
    static constexpr uint32_t kTxBytes =
        (uint32_t)(kTileRows * raw_row_bytes<WBITS>() + kMaxN * kStageK + kBlocksPerStage * kMaxN * 8);
    static constexpr int kTmemCols = kNAcc * kMaxN;
};

struct GemmParams {
    int mode;  // 0: gate/up (units carry the matrix), 1: down
    int K, nbK, nstage;
    int H, I;
    int prows_cap;
    const TcUnit* units;
    const int32_t* ctrl;  // plan results
    int n_units_idx;      // index of the unit count in ctrl
    int32_t* counter;     // unit counter (zeroed by the plan)
    const int32_t* row_slot;
    const float* s_r0;  // row scales: routed gate (or down), routed up, shared gate (or down), shared up
    const float* s_r1;
    const float* s_s0;
    const float* s_s1;
    float* gu;  // gate/up: [2][prows_cap][I]
    float* y;   // down: [slots][H]
    int32_t* err;
    const int* wide;   // some row's block scales spread too far for the digit planes
    const double* pe;  // digit-plane GEMM: 2^E of each padded row
};

// Exact fp64 of an int32: the 32 bits (offset by 2^31) become the low
// mantissa bits of 2^52, and the bias is subtracted.
__device__ __forceinline__ double exact_i2d(uint32_t v) {
    return __dsub_rn(__hiloint2double(0x43300000, (int)(v ^ 0x80000000u)), 4503601774854144.0);
}

template <int WBITS>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap w_r0, const __grid_constant__ CUtensorMap w_r1,
              const __grid_constant__ CUtensorMap w_s0, const __grid_constant__ CUtensorMap w_s1,
              const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap dmap,
              const GemmParams p) {
    if (!*p.wide) return;  // the digit-plane GEMM does this call's work
    using L = GemmSmem<WBITS>;
    constexpr int S = L::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ctl = sm + S * L::kStageBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
    uint64_t* conv = full + S;
    uint64_t* empty = conv + S;
    uint64_t* accf = empty + S;
    uint64_t* acce = accf + kNAcc;
    int* meta = reinterpret_cast<int*>(acce + kNAcc);  // [S][2]: unit (-1: end), stage of the unit
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(meta + 2 * S);
    auto stage = [&](int s) { return sm + s * L::kStageBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], kConvWarps);
            mbar_init(&empty[s], 1 + kEpiWarps);
        }
        for (int a = 0; a < kNAcc; ++a) {
            mbar_init(&accf[a], 1);
            mbar_init(&acce[a], kEpiWarps);
        }
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, L::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int n_units = p.ctrl[p.n_units_idx];

    if (warp == kProdWarp) {
        // ---------------- producer ----------------
        if (lane == 0) {
            tma_prefetch_map(&w_r0);
            tma_prefetch_map(&w_r1);
            tma_prefetch_map(&w_s0);
            tma_prefetch_map(&w_s1);
            tma_prefetch_map(&xmap);
            tma_prefetch_map(&dmap);
            int s = 0;
            uint32_t ph = 0;
            int unit = atomicAdd(p.counter, 1), kstep = 0;
            TcUnit u = unit < n_units ? p.units[unit] : TcUnit{0, 0, 0, 0};
            while (true) {
                if (!mbar_wait_ns(&empty[s], ph ^ 1u, kGemmWaitNs)) {
                    set_error(p.err, kErrTimeout);
                    break;
                }
                if (unit >= n_units) {
                    meta[2 * s] = -1;
                    meta[2 * s + 1] = 0;
                    mbar_arrive(&full[s]);
                    break;
                }
                meta[2 * s] = unit;
                meta[2 * s + 1] = kstep;
                mbar_arrive_expect_tx(&full[s], L::kTxBytes);
                uint8_t* st = stage(s);
                const bool sh = (u.info & kUnitShared) != 0, up = (u.info & kUnitUp) != 0;
                const CUtensorMap* wm = sh ? (up ? &w_s1 : &w_s0) : (up ? &w_r1 : &w_r0);
                tma_load_2d(WBITS == 8 ? st + L::kA : st + L::kRaw, wm, kstep * raw_row_bytes<WBITS>(), u.wrow0,
                            &full[s]);
                tma_load_2d(st + L::kX, &xmap, kstep * kStageK, u.prow0, &full[s]);
                tma_load_2d(st + L::kD, &dmap, u.prow0, kstep * kBlocksPerStage, &full[s]);
                if (++kstep == p.nstage) {
                    kstep = 0;
                    unit = atomicAdd(p.counter, 1);
                    if (unit < n_units) u = p.units[unit];
                }
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int s = 0, a = 0, cur = -1;
            uint32_t ph = 0, aph = 0, idesc = 0;
            bool ok = true;
            while (ok) {
                if (!mbar_wait_ns(&full[s], ph, kGemmWaitNs)) {
                    set_error(p.err, kErrTimeout);
                    break;
                }
                const int unit = meta[2 * s];
                if (unit < 0) break;
                const int kstep = meta[2 * s + 1];
                if (WBITS != 8 && !mbar_wait_ns(&conv[s], ph, kGemmWaitNs)) {
                    set_error(p.err, kErrTimeout);
                    break;
                }
                if (unit != cur) {
                    const int nt = p.units[unit].ntok;
                    idesc = idesc_i8((nt + 15) & ~15);
                    cur = unit;
                }
                tc_fence_after_sync();
                uint8_t* st = stage(s);
                const uint64_t xdsc = desc_k128_sw128(st + L::kX);
                const uint64_t adsc = desc_k128_sw128(st + L::kA);
#pragma unroll 1
                for (int j = 0; j < kBlocksPerStage; ++j) {
                    if (kstep * kBlocksPerStage + j >= p.nbK) break;
                    if (!mbar_wait_ns(&acce[a], aph ^ 1u, kGemmWaitNs)) {
                        set_error(p.err, kErrTimeout);
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    mma_i8(tmem + (uint32_t)(a * kMaxN), adsc + 2 * j, xdsc + 2 * j, idesc, false);
                    mma_commit(&accf[a]);
                    if (++a == kNAcc) {
                        a = 0;
                        aph ^= 1u;
                    }
                }
                mma_commit(&empty[s]);
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        __syncwarp();
    } else if (warp >= kEpiWarps) {
        // ---------------- widening ----------------
        if constexpr (WBITS != 8) {
            const int r0 = threadIdx.x - kEpiWarps * 32;  // rows r0 and r0 + 64 of the tile
            int s = 0;
            uint32_t ph = 0;
            while (true) {
                if (!mbar_wait_ns(&full[s], ph, kGemmWaitNs)) {
                    set_error(p.err, kErrTimeout);
                    break;
                }
                if (meta[2 * s] < 0) break;
                uint8_t* st = stage(s);
                widen_row<WBITS>(st + L::kRaw, st + L::kA, r0);
                widen_row<WBITS>(st + L::kRaw, st + L::kA, r0 + 64);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&conv[s]);
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int q = warp & 3, qt = warp >> 2;
        const uint32_t tlane = (uint32_t)(32 * q) << 16;
        int s = 0, a = 0;
        uint32_t ph = 0, aph = 0;
        TcUnit u{0, 0, 0, 0};
        double acc[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = 0.0;
        bool ok = true;
        while (ok) {
            if (!mbar_wait_ns(&full[s], ph, kGemmWaitNs)) {
                set_error(p.err, kErrTimeout);
                break;
            }
            const int unit = meta[2 * s];
            if (unit < 0) break;
            const int kstep = meta[2 * s + 1];
            if (kstep == 0) {
                u = p.units[unit];
#pragma unroll
                for (int c = 0; c < 16; ++c) acc[c] = 0.0;
            }
            const bool active = 16 * qt < u.ntok;  // the same in the whole warp
            const double* dt = reinterpret_cast<const double*>(stage(s) + L::kD);
#pragma unroll 1
            for (int j = 0; j < kBlocksPerStage; ++j) {
                if (kstep * kBlocksPerStage + j >= p.nbK) break;
                if (!mbar_wait_ns(&accf[a], aph, kGemmWaitNs)) {
                    set_error(p.err, kErrTimeout);
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                if (active) {
                    uint32_t v[16];
                    tmem_ld16(tmem + tlane + (uint32_t)(a * kMaxN + 16 * qt), v);
                    tmem_wait_ld();
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acce[a]);
                    const double2* d2 = reinterpret_cast<const double2*>(dt + j * kMaxN + 16 * qt);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const double2 dd = d2[i];
                        acc[2 * i] = __fma_rn(dd.x, exact_i2d(v[2 * i]), acc[2 * i]);
                        acc[2 * i + 1] = __fma_rn(dd.y, exact_i2d(v[2 * i + 1]), acc[2 * i + 1]);
                    }
                } else {
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&acce[a]);
                }
                if (++a == kNAcc) {
                    a = 0;
                    aph ^= 1u;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (ok && kstep == p.nstage - 1 && active) {
                const int tile = u.info & 0xFFFF;
                const bool sh = (u.info & kUnitShared) != 0, up = (u.info & kUnitUp) != 0;
                const int rl = 32 * q + lane;
                const float* sc = sh ? (up ? p.s_s1 : p.s_s0) : (up ? p.s_r1 : p.s_r0);
                const double sr = (double)__ldg(sc + u.wrow0 + rl);
                const int r = tile * kTileRows + rl;  // output row of this thread
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int col = 16 * qt + c;
                    if (col >= u.ntok) continue;
                    const int prow = u.prow0 + col;
                    const float v = __double2float_rn(__dmul_rn(sr, acc[c]));
                    if (p.mode == 0) {
                        p.gu[((int64_t)(up ? p.prows_cap : 0) + prow) * p.I + r] = v;
                    } else {
                        const int slot = p.row_slot[prow];
                        if (slot >= 0) p.y[(int64_t)slot * p.H + r] = v;
                    }
                }
            }
            if (++s == S) {
                s = 0;
                ph ^= 1u;
            }
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == kMmaWarp) tmem_dealloc(tmem, L::kTmemCols);
}

// ---------------------------------------------------------------------------
// Grouped GEMM on the digit planes (persistent, one CTA per SM)
// ---------------------------------------------------------------------------
// Per unit (128 weight rows x a chunk of nt <= kChunk tokens) one kind::i8
// MMA per 32 codes of K with M = 128 and N = kPlanes * nt16 columns: column
// 5 c + p is token c's plane p (the plane tensor is [rows][kPlanes][K], so a
// chunk's planes are kPlanes * nt consecutive rows).  The accumulator sums
// the whole K in int32; at the unit's end
//   acc = 2^E_c (D_0 + 2^8 D_1 + 2^16 D_2 + 2^24 D_3 + 2^32 D_4)
// is formed exactly in int64 (a double while it stays below 2^53), and the
// output is fp32(s_row * acc) in fp64, as the oracle rounds it.
// warps 0-3, 10-13  epilogue (warp w: TMEM lanes 32 (w % 4) .. + 31 = its 32
//            rows; warps 0-3 take tokens 0-7 of each 16-token group, 10-13
//            tokens 8-15)
// warps 4-7  widening of the packed int4 / int2 staging rows (one row per
//            thread; codes at the top of their bytes, see widen_row_top)
// warp 8     producer: TMA per stage of the weight rows and of the chunk's
//            planes (box of 80, 160 or 240 rows)
// warp 9     MMA: two accumulators of 256 TMEM columns, alternating units;
//            its stage waits suspend for at most 32 ns at a time
//            (mbar_wait_short): with the default suspend the tensor pipe sat
//            idle long after a stage's operands had landed
// Every wait is bounded by the global timer and records kErrTimeout.
constexpr int kDpEpiWarps = 4;  // of each of the two epilogue sets
constexpr int kDpConvWarps = 4;
constexpr int kDpWidenParts = kDpConvWarps * 32 / kTileRows;  // threads per widened row
static_assert(kDpWidenParts * kTileRows == kDpConvWarps * 32, "whole rows per widening pass");
constexpr int kDpProdWarp = kDpEpiWarps + kDpConvWarps;
constexpr int kDpMmaWarp = kDpProdWarp + 1;
constexpr int kDpEpiWarps2 = kDpMmaWarp + 1;  // the second epilogue set: warps 10-13
constexpr int kDpThreads = (kDpEpiWarps2 + kDpEpiWarps) * 32;
constexpr int kDpAccCols = 256;

template <int WBITS>
struct DpSmem {
    static constexpr int kRawTile = WBITS == 8 ? 0 : kTileRows * raw_row_bytes<WBITS>();
    static constexpr int kA = 0;                                   // widened tile (int8: the TMA target)
    static constexpr int kB = kTileBytes;                          // planes [kPlanes * kChunk][128]
    static constexpr int kRaw = kB + kPlanes * kChunk * kStageK;  // packed staging tile
    static constexpr int kStageBytes = (kRaw + kRawTile + 1023) & ~1023;
    static constexpr int kCtrl = 1024;
    static constexpr int kStagesFit = (224 * 1024 - kCtrl - 1024) / kStageBytes;
    static constexpr int kStages = kStagesFit < 6 ? kStagesFit : 6;
    static constexpr int kBytes = kStages * kStageBytes + kCtrl + 1024;  // + alignment slack
    static constexpr uint32_t kWeightTx = (uint32_t)(kTileRows * raw_row_bytes<WBITS>());
};

// Tokens of a unit -> groups of 16 (1..3): which plane map, and N / 80
__device__ __forceinline__ int nt_groups(int ntok) { return (ntok + 15) >> 4; }

template <int WBITS>
__global__ void __launch_bounds__(kDpThreads, 1)
    k_tc_gemm_dp(const __grid_constant__ CUtensorMap w_r0, const __grid_constant__ CUtensorMap w_r1,
                 const __grid_constant__ CUtensorMap w_s0, const __grid_constant__ CUtensorMap w_s1,
                 const __grid_constant__ CUtensorMap b16, const __grid_constant__ CUtensorMap b32,
                 const __grid_constant__ CUtensorMap b48, const GemmParams p) {
    if (*p.wide) return;  // the fp64-epilogue GEMM does this call's work
    using L = DpSmem<WBITS>;
    constexpr int S = L::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ctl = sm + S * L::kStageBytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
    uint64_t* conv = full + S;
    uint64_t* empty = conv + S;
    uint64_t* accf = empty + S;  // [2] the accumulator's unit is complete (MMA commit)
    uint64_t* acce = accf + 2;   // [2] the epilogue has read the accumulator
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
    auto stage = [&](int s) { return sm + s * L::kStageBytes; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], kDpConvWarps);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&accf[a], 1);
            mbar_init(&acce[a], 2 * kDpEpiWarps);
        }
        fence_barrier_init();
    }
    if (warp == kDpMmaWarp) {
        tmem_alloc(tmem_slot, 2 * kDpAccCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // Units are dealt round-robin: this CTA's are blockIdx.x, + gridDim.x, ...
    // Every unit is nstage stages of the same work, so the deal is as even as
    // a counter's, and each role walks the sequence on its own (no hand-over
    // of unit ids, no atomics).
    const int n_units = p.ctrl[p.n_units_idx];
    const int u0 = blockIdx.x, du = gridDim.x;
    const int my_units = u0 < n_units ? (n_units - 1 - u0) / du + 1 : 0;

    if (warp == kDpProdWarp) {
        // ---------------- producer ----------------
        if (lane == 0 && my_units > 0) {
            tma_prefetch_map(&w_r0);
            tma_prefetch_map(&w_r1);
            tma_prefetch_map(&w_s0);
            tma_prefetch_map(&w_s1);
            tma_prefetch_map(&b16);
            tma_prefetch_map(&b32);
            tma_prefetch_map(&b48);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            TcUnit u = p.units[u0];
            for (int unit = u0; ok && unit < n_units; unit += du) {
                // the next unit's description is in flight during this one
                const TcUnit un = unit + du < n_units ? p.units[unit + du] : u;
                const int ng = nt_groups(u.ntok);
                const uint32_t tx = L::kWeightTx + (uint32_t)(kPlanes * 16 * ng * kStageK);
                const bool sh = (u.info & kUnitShared) != 0, up = (u.info & kUnitUp) != 0;
                const CUtensorMap* wm = sh ? (up ? &w_s1 : &w_s0) : (up ? &w_r1 : &w_r0);
                const CUtensorMap* bm = ng == 1 ? &b16 : ng == 2 ? &b32 : &b48;
                for (int kstep = 0; kstep < p.nstage; ++kstep) {
                    if (!mbar_wait_ns(&empty[s], ph ^ 1u, kGemmWaitNs)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], tx);
                    uint8_t* st = stage(s);
                    tma_load_2d(WBITS == 8 ? st + L::kA : st + L::kRaw, wm, kstep * raw_row_bytes<WBITS>(), u.wrow0,
                                &full[s]);
                    tma_load_2d(st + L::kB, bm, kstep * kStageK, u.prow0 * kPlanes, &full[s]);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                u = un;
            }
            if (!ok) set_error(p.err, kErrTimeout);
        }
        __syncwarp();
    } else if (warp == kDpMmaWarp) {
        // ---------------- MMA issuer ----------------
        if (lane == 0 && my_units > 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int ntok = p.units[u0].ntok;
            for (int unit = u0, nu = 0; ok && unit < n_units; unit += du, ++nu) {
                const int ntok_next = unit + du < n_units ? p.units[unit + du].ntok : 0;
                // the unit takes the next accumulator once the epilogue has
                // read that accumulator's previous unit
                const int buf = nu & 1;
                if (nu >= 2 && !mbar_wait_short(&acce[buf], ((nu >> 1) - 1) & 1, kGemmWaitNs)) {
                    ok = false;
                    break;
                }
                const uint32_t idesc = idesc_i8(kPlanes * 16 * nt_groups(ntok));
                const uint32_t acc = tmem + (uint32_t)(buf * kDpAccCols);
                for (int kstep = 0; kstep < p.nstage; ++kstep) {
                    if (!mbar_wait_short(&full[s], ph, kGemmWaitNs) ||
                        (WBITS != 8 && !mbar_wait_short(&conv[s], ph, kGemmWaitNs))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    uint8_t* st = stage(s);
                    const uint64_t bdsc = desc_k128_sw128(st + L::kB);
                    const uint64_t adsc = desc_k128_sw128(st + L::kA);
#pragma unroll
                    for (int j = 0; j < kBlocksPerStage; ++j)
                        if (kstep * kBlocksPerStage + j < p.nbK)
                            mma_i8(acc, adsc + 2 * j, bdsc + 2 * j, idesc, kstep > 0 || j > 0);
                    mma_commit(&empty[s]);
                    if (++s == S) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&accf[buf]);
                ntok = ntok_next;
            }
            if (!ok) set_error(p.err, kErrTimeout);
        }
        __syncwarp();
    } else if (warp >= kDpEpiWarps && warp < kDpEpiWarps + kDpConvWarps) {
        // ---------------- widening ----------------
        if constexpr (WBITS != 8) {
            // thread i widens part i / 128 of row i % 128 of the tile
            const int ci = threadIdx.x - kDpEpiWarps * 32;
            const int crow = ci % kTileRows, cpart = ci / kTileRows;
            const int n_st = my_units * p.nstage;
            int s = 0;
            uint32_t ph = 0;
            for (int i = 0; i < n_st; ++i) {
                if (!mbar_wait_ns(&full[s], ph, kGemmWaitNs)) {
                    set_error(p.err, kErrTimeout);
                    break;
                }
                uint8_t* st = stage(s);
                widen_row_top<WBITS, kDpWidenParts>(st + L::kRaw, st + L::kA, crow, cpart);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&conv[s]);
                if (++s == S) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else {
        // ---------------- epilogue ----------------
        const int quad = warp & 3, part = warp >= kDpEpiWarps2 ? 1 : 0;  // TMEM lane quarter; tokens 8 part ..
        const uint32_t tlane = (uint32_t)(32 * quad) << 16;
        const int rl = 32 * quad + lane;  // the thread's row in the tile
        for (int unit = u0, nu = 0; unit < n_units; unit += du, ++nu) {
            const int buf = nu & 1;
            const uint32_t par = (uint32_t)(nu >> 1) & 1u;
            // the unit's description, row scale, 2^E and (down) slots are
            // loaded while its MMAs run; one token per lane (kChunk <= 64)
            const TcUnit u = p.units[unit];
            const int tile = u.info & 0xFFFF;
            const bool sh = (u.info & kUnitShared) != 0, up = (u.info & kUnitUp) != 0;
            const float* sc = sh ? (up ? p.s_s1 : p.s_s0) : (up ? p.s_r1 : p.s_r0);
            const double sr = (double)__ldg(sc + u.wrow0 + rl);
            const int r = tile * kTileRows + rl;  // output row of this thread
            const int ng = nt_groups(u.ntok);
            const bool ina = lane < u.ntok, inb = lane + 32 < u.ntok;
            const double pea = ina ? __ldg(p.pe + u.prow0 + lane) : 0.0;
            const double peb = inb ? __ldg(p.pe + u.prow0 + lane + 32) : 0.0;
            const int sla = (p.mode == 1 && ina) ? __ldg(p.row_slot + u.prow0 + lane) : -1;
            const int slb = (p.mode == 1 && inb) ? __ldg(p.row_slot + u.prow0 + lane + 32) : -1;
            if (!mbar_wait_ns(&accf[buf], par, kGemmWaitNs)) {
                set_error(p.err, kErrTimeout);
                break;
            }
            tc_fence_after_sync();
            for (int g = 0; g < ng; ++g) {
                // this set's 8 tokens of the group: accumulator columns
                // 80 g + 40 part .. + 39 (column 5 c + p: token c's plane p)
                if (16 * g + 8 * part >= u.ntok) break;  // the same in the whole warp
                uint32_t v[kPlanes * 8];
                const uint32_t col = (uint32_t)(buf * kDpAccCols + kPlanes * 16 * g + kPlanes * 8 * part);
                {
                    uint32_t a16[16], b16[16], c8[8];
                    tmem_ld16(tmem + tlane + col, a16);
                    tmem_ld16(tmem + tlane + col + 16, b16);
                    tmem_ld8(tmem + tlane + col + 32, c8);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        v[k] = a16[k];
                        v[16 + k] = b16[k];
                    }
#pragma unroll
                    for (int k = 0; k < 8; ++k) v[32 + k] = c8[k];
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int tk = 16 * g + 8 * part + c;
                    if (tk >= u.ntok) break;  // the same in the whole warp
                    const double pe = __shfl_sync(kFull, tk < 32 ? pea : peb, tk & 31);
                    const int slot = __shfl_sync(kFull, tk < 32 ? sla : slb, tk & 31);
                    const int64_t sum = (int64_t)(int)v[kPlanes * c] + ((int64_t)(int)v[kPlanes * c + 1] << 8) +
                                        ((int64_t)(int)v[kPlanes * c + 2] << 16) +
                                        ((int64_t)(int)v[kPlanes * c + 3] << 24) +
                                        ((int64_t)(int)v[kPlanes * c + 4] << 32);
                    // every plane's dot is 2^kWidenShift times the exact one (the weights
                    // were widened to the top of their bytes): an exact shift, then 2^E
                    const double accd = __dmul_rn(__ll2double_rn(sum >> kWidenShift<WBITS>), pe);
                    const float val = __double2float_rn(__dmul_rn(sr, accd));
                    if (p.mode == 0) {
                        p.gu[((int64_t)(up ? p.prows_cap : 0) + u.prow0 + tk) * p.I + r] = val;
                    } else if (slot >= 0) {
                        p.y[(int64_t)slot * p.H + r] = val;
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acce[buf]);
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == kDpMmaWarp) tmem_dealloc(tmem, 2 * kDpAccCols);
}

// SwiGLU and Q8_0 of h, one CTA per padded row, four consecutive elements a
// thread: h = silu(g) * u evaluated in fp64 and rounded to fp32, then Q8_0;
// the codes and scales go to the slot's h (hq, hd), to the row's codes and
// transposed fp64 scales (hg, hdT: the fp64-epilogue GEMM's operands) and,
// as in k_tc_quantize, to the row's digit planes [5][inter] with 2^E in peh
// (a row too wide for the planes sets *wide).  Padding rows: zero planes and
// scales.  inter is a multiple of 128 (a warp's elements are all in the row
// or all past it).
__global__ void __launch_bounds__(kQuantThreads) k_tc_swiglu(const float* __restrict__ gu, int I, int prows_cap,
                                                             const int32_t* __restrict__ row_slot,
                                                             const int32_t* __restrict__ ctrl, int8_t* __restrict__ hg,
                                                             double* __restrict__ hdT, int8_t* __restrict__ hq,
                                                             float* __restrict__ hd, int8_t* __restrict__ hp,
                                                             double* __restrict__ peh, int* wide) {
    __shared__ uint32_t s_m[kMaxQuantCols / 32];
    __shared__ int s_e[kMaxQuantCols / 32];
    __shared__ int s_red[2 * kQuantThreads / 32];
    const int q = blockIdx.x, lane = threadIdx.x & 31;
    if (q >= ctrl[2]) return;
    const int nbI = I / 32;
    const int slot = row_slot[q];
    int8_t* dst = hp + (int64_t)q * kPlanes * I;
    if (slot < 0) {  // a padding row
        for (int b = threadIdx.x; b < nbI; b += kQuantThreads) hdT[(int64_t)b * prows_cap + q] = 0.0;
        uint4* d16 = reinterpret_cast<uint4*>(dst);
        for (int i = threadIdx.x; i < kPlanes * I / 16; i += kQuantThreads) d16[i] = make_uint4(0u, 0u, 0u, 0u);
        if (threadIdx.x == 0) peh[q] = 0.0;
        return;
    }
    const float4* gr = reinterpret_cast<const float4*>(gu + (int64_t)q * I);
    const float4* ur = reinterpret_cast<const float4*>(gu + ((int64_t)prows_cap + q) * I);
    uint32_t codes[kQuadIters];
    float4 g = 4 * threadIdx.x < I ? gr[threadIdx.x] : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 u = 4 * threadIdx.x < I ? ur[threadIdx.x] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < kQuadIters; ++j) {
        const int v = threadIdx.x + j * kQuantThreads, i = 4 * v;
        if (i >= I) break;
        // the next pass's loads in flight while this one is computed
        const bool nx = i + kQuadSpan < I;
        const float4 gn = nx ? gr[v + kQuantThreads] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 un = nx ? ur[v + kQuantThreads] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float gv[4] = {g.x, g.y, g.z, g.w}, uv[4] = {u.x, u.y, u.z, u.w};
        float h[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const double gd = (double)gv[e];
            h[e] = __double2float_rn(__dmul_rn(__ddiv_rn(gd, __dadd_rn(1.0, exp(-gd))), (double)uv[e]));
        }
        float d;
        const uint32_t c = q8_0_quad(h, d);
        codes[j] = c;
        *reinterpret_cast<uint32_t*>(hg + (int64_t)q * I + i) = c;
        *reinterpret_cast<uint32_t*>(hq + (int64_t)slot * I + i) = c;
        if ((lane & 7) == 0) {
            const int b = i >> 5;
            hdT[(int64_t)b * prows_cap + q] = (double)d;
            hd[(int64_t)slot * nbI + b] = d;
            f32_mant_exp(d, s_m[b], s_e[b]);
        }
        g = gn;
        u = un;
    }
    row_planes_quad(codes, s_m, s_e, I, s_red, dst, peh + q, wide);
}

}  // namespace tc

// ---------------------------------------------------------------------------
// Host side of the batched path
// ---------------------------------------------------------------------------
bool tc_path_supported(const moe_config& c, int T) {
    if (T < kTcMinTokens) return false;
    if (c.hidden % tc::kTileRows || c.inter % tc::kTileRows) return false;
    // the quantisers hold a row's codes in shared memory
    if (c.hidden > tc::kMaxQuantCols || c.inter > tc::kMaxQuantCols) return false;
    return c.wbits == 8 || c.wbits == 4 || c.wbits == 2;
}

TcSizes tc_sizes(const moe_config& c, int T) {
    const int64_t pairs = (int64_t)T * c.top_k, slots = pairs + (int64_t)T * c.n_shared;
    const int64_t entries = (c.n_experts < pairs ? c.n_experts : pairs) + c.n_shared;
    TcSizes z;
    z.prows_cap = (int)(((slots + 15 * entries) + 63) / 64 * 64 + 64);
    const int64_t chunks = (slots + tc::kChunk - 1) / tc::kChunk + entries;
    z.units_gu_cap = (int)(2 * chunks * (c.inter / tc::kTileRows));
    z.units_dn_cap = (int)(chunks * (c.hidden / tc::kTileRows));
    return z;
}

cudaError_t launch_tc_prepare(const TcArgs& a, cudaStream_t s) {
    const moe_config& c = *a.ex.cfg;
    tc::PlanParams pp;
    pp.T = a.ex.T; pp.k = c.top_k; pp.E = c.n_experts; pp.ns = c.n_shared; pp.I = c.inter; pp.H = c.hidden;
    pp.prows_cap = a.sz.prows_cap; pp.units_gu_cap = a.sz.units_gu_cap; pp.units_dn_cap = a.sz.units_dn_cap;
    pp.offsets = a.ex.offsets; pp.perm = a.ex.perm; pp.active = a.ex.active;
    pp.units_gu = static_cast<tc::TcUnit*>(a.units_gu);
    pp.units_dn = static_cast<tc::TcUnit*>(a.units_dn);
    pp.row_tok = a.row_tok; pp.row_slot = a.row_slot; pp.ctrl = a.ctrl; pp.err = a.ex.err;
    tc::k_tc_plan<<<tc::kPlanCtas, tc::kPlanThreads, 0, s>>>(pp);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int grid = (a.sz.prows_cap + 7) / 8;
    tc::k_tc_gather<<<grid, 256, 0, s>>>(a.ex.xq, a.ex.xd, a.xpt, a.pet, a.xwide, c.hidden, a.sz.prows_cap,
                                         a.row_tok, a.ctrl, a.xg, a.xdT, a.xp, a.pex);
    return cudaGetLastError();
}

cudaError_t launch_tc_quantize(const float* x, int T, int H, int8_t* xq, float* xd, int8_t* xpt, double* pet,
                               int* xwide, cudaStream_t s) {
    if (T == 0) return cudaSuccess;
    tc::k_tc_quantize<<<T, tc::kQuantThreads, 0, s>>>(x, H, xq, xd, xpt, pet, xwide);
    return cudaGetLastError();
}

namespace tc {

template <int WBITS>
static cudaError_t launch_gemm_t(const CUtensorMap (&m)[6], const GemmParams& gp, cudaStream_t s) {
    using L = GemmSmem<WBITS>;
    static_assert(L::kStages >= 2, "at least two pipeline stages");
    static bool attr_done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!attr_done[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(k_tc_gemm<WBITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    k_tc_gemm<WBITS><<<device_info().sm_count, kGemmThreads, L::kBytes, s>>>(m[0], m[1], m[2], m[3], m[4], m[5], gp);
    return cudaGetLastError();
}

static cudaError_t launch_gemm(int wbits, const CUtensorMap (&m)[6], const GemmParams& gp, cudaStream_t s) {
    if (wbits == 4) return launch_gemm_t<4>(m, gp, s);
    if (wbits == 2) return launch_gemm_t<2>(m, gp, s);
    return launch_gemm_t<8>(m, gp, s);
}

template <int WBITS>
static cudaError_t launch_gemm_dp_t(const CUtensorMap (&m)[7], const GemmParams& gp, cudaStream_t s) {
    using L = DpSmem<WBITS>;
    static_assert(L::kStages >= 2, "at least two pipeline stages");
    static bool attr_done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!attr_done[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(k_tc_gemm_dp<WBITS>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
        if (e != cudaSuccess) return e;
        attr_done[dev] = true;
    }
    k_tc_gemm_dp<WBITS><<<device_info().sm_count, kDpThreads, L::kBytes, s>>>(m[0], m[1], m[2], m[3], m[4], m[5],
                                                                               m[6], gp);
    return cudaGetLastError();
}

static cudaError_t launch_gemm_dp(int wbits, const CUtensorMap (&m)[7], const GemmParams& gp, cudaStream_t s) {
    if (wbits == 4) return launch_gemm_dp_t<4>(m, gp, s);
    if (wbits == 2) return launch_gemm_dp_t<2>(m, gp, s);
    return launch_gemm_dp_t<8>(m, gp, s);
}

// Maps of a plane tensor [prows_cap * kPlanes][K] with boxes of 80, 160 and
// 240 rows (the chunk's planes at 16, 32 or 48 tokens), 128-byte swizzle.
static cudaError_t encode_planes(CUtensorMap (&b)[3], const int8_t* planes, int K, int prows_cap) {
    for (int g = 0; g < 3; ++g) {
        const cudaError_t e = encode_2d(&b[g], planes, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)K,
                                        (uint64_t)prows_cap * kPlanes, (uint64_t)K, kStageK,
                                        (uint32_t)(kPlanes * 16 * (g + 1)), CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Token-side maps of a GEMM: codes [prows_cap][K] (128-byte swizzle) and block
// scales [K/32][prows_cap] fp64.
static cudaError_t encode_tokens(CUtensorMap* codes, CUtensorMap* scales, const void* q, const double* dT, int K,
                                 int prows_cap) {
    cudaError_t e = encode_2d(codes, q, CU_TENSOR_MAP_DATA_TYPE_UINT8, (uint64_t)K, (uint64_t)prows_cap,
                              (uint64_t)K, kStageK, kMaxN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    return encode_2d(scales, dT, CU_TENSOR_MAP_DATA_TYPE_FLOAT64, (uint64_t)prows_cap, (uint64_t)(K / 32),
                     (uint64_t)prows_cap * 8, kMaxN, kBlocksPerStage, CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace tc

cudaError_t launch_tc_experts(const TcArgs& a, cudaStream_t s, cudaEvent_t const* ev) {
    using namespace tc;
    const moe_config& c = *a.ex.cfg;
    const int H = c.hidden, I = c.inter, E = c.n_experts, wb = c.wbits;
    const moe_experts& R = a.ex.routed;
    const moe_experts& Sh = c.n_shared ? a.ex.shared : a.ex.routed;
    const int64_t sh_rows_gu = c.n_shared ? I : (int64_t)E * I, sh_rows_dn = c.n_shared ? H : (int64_t)E * H;
    cudaError_t e;
    // gate/up: weights [E * I][H], tokens xg / xdT -> g, u per padded row
    {
        CUtensorMap m[6];
        if ((e = encode_weights(&m[0], R.w_gate, (int64_t)E * I, H, wb)) != cudaSuccess) return e;
        if ((e = encode_weights(&m[1], R.w_up, (int64_t)E * I, H, wb)) != cudaSuccess) return e;
        if ((e = encode_weights(&m[2], Sh.w_gate, sh_rows_gu, H, wb)) != cudaSuccess) return e;
        if ((e = encode_weights(&m[3], Sh.w_up, sh_rows_gu, H, wb)) != cudaSuccess) return e;
        if ((e = encode_tokens(&m[4], &m[5], a.xg, a.xdT, H, a.sz.prows_cap)) != cudaSuccess) return e;
        GemmParams gp{};
        gp.mode = 0; gp.K = H; gp.nbK = H / 32; gp.nstage = (H + kStageK - 1) / kStageK; gp.H = H; gp.I = I;
        gp.prows_cap = a.sz.prows_cap; gp.units = static_cast<const TcUnit*>(a.units_gu); gp.ctrl = a.ctrl;
        gp.n_units_idx = 0; gp.counter = a.ctrl + 3; gp.row_slot = a.row_slot;
        gp.s_r0 = R.s_gate; gp.s_r1 = R.s_up; gp.s_s0 = Sh.s_gate; gp.s_s1 = Sh.s_up;
        gp.gu = a.gu; gp.y = a.ex.y; gp.err = a.ex.err;
        gp.wide = a.xwide; gp.pe = a.pex;
        CUtensorMap md[7] = {m[0], m[1], m[2], m[3]};
        if ((e = encode_planes(*reinterpret_cast<CUtensorMap(*)[3]>(&md[4]), a.xp, H, a.sz.prows_cap)) != cudaSuccess)
            return e;
        // the digit-plane GEMM, or (a token too wide for the planes) the fp64 one
        if ((e = launch_gemm_dp(wb, md, gp, s)) != cudaSuccess) return e;
        if ((e = launch_gemm(wb, m, gp, s)) != cudaSuccess) return e;
        // the "gate_up" phase ends with the GEMM; SwiGLU opens the "down" phase
        if (ev && (e = record_event(ev[0], s)) != cudaSuccess) return e;
        k_tc_swiglu<<<a.sz.prows_cap, kQuantThreads, 0, s>>>(a.gu, I, a.sz.prows_cap, a.row_slot, a.ctrl, a.hg, a.hdT,
                                                            a.ex.hq, a.ex.hd, a.hp, a.peh, a.hwide);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // down: weights [E * H][I], h codes hg / hdT -> y per slot
    {
        CUtensorMap m[6];
        if ((e = encode_weights(&m[0], R.w_down, (int64_t)E * H, I, wb)) != cudaSuccess) return e;
        m[1] = m[0];
        if ((e = encode_weights(&m[2], Sh.w_down, sh_rows_dn, I, wb)) != cudaSuccess) return e;
        m[3] = m[2];
        if ((e = encode_tokens(&m[4], &m[5], a.hg, a.hdT, I, a.sz.prows_cap)) != cudaSuccess) return e;
        GemmParams gp{};
        gp.mode = 1; gp.K = I; gp.nbK = I / 32; gp.nstage = (I + kStageK - 1) / kStageK; gp.H = H; gp.I = I;
        gp.prows_cap = a.sz.prows_cap; gp.units = static_cast<const TcUnit*>(a.units_dn); gp.ctrl = a.ctrl;
        gp.n_units_idx = 1; gp.counter = a.ctrl + 4; gp.row_slot = a.row_slot;
        gp.s_r0 = R.s_down; gp.s_r1 = R.s_down; gp.s_s0 = Sh.s_down; gp.s_s1 = Sh.s_down;
        gp.gu = a.gu; gp.y = a.ex.y; gp.err = a.ex.err;
        gp.wide = a.hwide; gp.pe = a.peh;
        CUtensorMap md[7] = {m[0], m[1], m[2], m[3]};
        if ((e = encode_planes(*reinterpret_cast<CUtensorMap(*)[3]>(&md[4]), a.hp, I, a.sz.prows_cap)) != cudaSuccess)
            return e;
        if ((e = launch_gemm_dp(wb, md, gp, s)) != cudaSuccess) return e;
        if ((e = launch_gemm(wb, m, gp, s)) != cudaSuccess) return e;
        if (ev && (e = record_event(ev[1], s)) != cudaSuccess) return e;
    }
    if ((e = launch_combine(a.ex, s)) != cudaSuccess) return e;
    if (ev && (e = record_event(ev[2], s)) != cudaSuccess) return e;
    return cudaSuccess;
}

}  // namespace moe
