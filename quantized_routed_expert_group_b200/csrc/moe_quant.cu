// moe_quant.cu -- Q8_0 activation quantiser and per-row weight quantiser.
//
// Q8_0: GeekNews "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", §구현된 주요 기능
// (integer-dot kernel with Q8_0-style int8 activations); wpnews.pro "Colibri —
// รัน GLM-5.2 ...", kernel table.  Weight quantiser: same page, quantisation
// kernel bullet (int8 / packed int4 / packed int2, per-row scales) and the
// offline converter that dequantises the FP8 checkpoint with its 128 x 128
// block scales and requantises it per row (same bullet list; wpnews.pro
// converter list).
#include <cuda_fp16.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

// One warp per Q8_0 block of 32 values; 8 blocks per CTA, grid-stride.
__global__ void __launch_bounds__(256) k_quantize_q8_0(const float* __restrict__ x, int64_t nblk,
                                                       int8_t* __restrict__ q, float* __restrict__ d) {
    const int lane = threadIdx.x & 31;
    for (int64_t b = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); b < nblk; b += (int64_t)gridDim.x * 8) {
        const float v = x[b * kQBlock + lane];
        int8_t qq;
        float dd;
        q8_0_warp(v, qq, dd);
        q[b * kQBlock + lane] = qq;
        if (lane == 0) d[b] = dd;
    }
}

cudaError_t launch_quantize_q8_0(const float* x, int64_t n_rows, int cols, int8_t* q, float* d,
                                 cudaStream_t s) {
    const int64_t nblk = n_rows * (cols / kQBlock);
    if (nblk == 0) return cudaSuccess;
    const int64_t want = (nblk + 7) / 8;
    const int grid = (int)(want < 65535 * 8 ? want : 65535 * 8);
    k_quantize_q8_0<<<grid, 256, 0, s>>>(x, nblk, q, d);
    return cudaGetLastError();
}

// Row sources of the per-row quantiser: get(r, i) returns the fp32 values of
// row r at columns i .. i+3 (i a multiple of 4).
struct RowsF32 {  // plain fp32 rows [rows][cols]
    const float* w;
    int cols;
    __device__ __forceinline__ float4 get(int64_t r, int i) const {
        return *reinterpret_cast<const float4*>(w + r * cols + i);
    }
};

// FP8 E4M3 value of one code, from the format: 1 sign bit, 4 exponent bits
// with bias 7, 3 mantissa bits; exponent 0 is subnormal (m * 2^-9); S.1111.111
// is NaN; there are no infinities.  A normal code maps to the fp32 with
// exponent e - 7 + 127 and the 3 mantissa bits on top of its mantissa.
__device__ __forceinline__ float fp8_e4m3_value(uint32_t b) {
    const uint32_t e = (b >> 3) & 0xFu, m = b & 7u, sign = (b & 0x80u) << 24;
    if (e == 15u && m == 7u) return __uint_as_float(0x7FC00000u);
    if (e == 0u) return __uint_as_float(sign | __float_as_uint((float)m * 0.001953125f));
    return __uint_as_float(sign | ((e + 120u) << 23) | (m << 20));
}

struct RowsFp8Block {  // FP8 E4M3 rows [rows][cols] times their block scales
    const uint8_t* w8;
    const float* bs;  // [ceil(rows/block)][nbc]
    int cols, block, nbc;
    __device__ __forceinline__ float4 get(int64_t r, int i) const {
        const uint32_t b4 = *reinterpret_cast<const uint32_t*>(w8 + r * cols + i);
        const float sc = bs[(r / block) * nbc + i / block];  // block % 4 == 0: one block for the four
        return make_float4(__fmul_rn(fp8_e4m3_value(b4 & 0xFFu), sc), __fmul_rn(fp8_e4m3_value((b4 >> 8) & 0xFFu), sc),
                           __fmul_rn(fp8_e4m3_value((b4 >> 16) & 0xFFu), sc), __fmul_rn(fp8_e4m3_value(b4 >> 24), sc));
    }
};

// Per-row quantiser: one CTA per row.  s = amax / qmax, code =
// round-half-away(w * (1/s)) clamped to [-2^(b-1), qmax], packed two's
// complement with the lowest element in the lowest bits.
template <int WBITS, class Rows>
__global__ void __launch_bounds__(256) k_pack_rows(const Rows src, int64_t rows, int cols,
                                                   uint8_t* __restrict__ packed, float* __restrict__ scales) {
    constexpr int qmax = WBITS == 8 ? 127 : WBITS == 4 ? 7 : 1;
    constexpr float qminf = -(float)(1 << (WBITS - 1));
    __shared__ float red[8];
    __shared__ float s_is[2];
    const int64_t row_bytes = (int64_t)cols * WBITS / 8;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        float a = 0.0f;
        for (int i = threadIdx.x * 4; i < cols; i += blockDim.x * 4) {
            const float4 v = src.get(r, i);
            a = fmaxf(a, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
        __syncthreads();
        if (threadIdx.x == 0) {
            float m = red[0];
            for (int i = 1; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
            float sc = 0.0f, is = 0.0f;
            if (m >= FLT_MIN) {
                sc = __fdiv_rn(m, (float)qmax);
                is = __fdiv_rn(1.0f, sc);
            }
            scales[r] = sc;
            s_is[0] = is;
            s_is[1] = sc;
        }
        __syncthreads();
        const float is = s_is[0];
        const bool zero = !(s_is[1] > 0.0f);
        // each thread packs groups of 32 codes
        for (int g = threadIdx.x; g < cols / 32; g += blockDim.x) {
            int codes[32];
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 v = src.get(r, 32 * g + i);
                const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float c = roundf(__fmul_rn(vv[j], is));
                    c = fminf(fmaxf(c, qminf), (float)qmax);
                    codes[i + j] = zero ? 0 : (int)c;
                }
            }
            uint8_t* dst = packed + r * row_bytes + (int64_t)g * 32 * WBITS / 8;
            if constexpr (WBITS == 8) {
                uint32_t out[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    out[k] = (uint32_t)(codes[4 * k] & 0xFF) | ((uint32_t)(codes[4 * k + 1] & 0xFF) << 8) |
                             ((uint32_t)(codes[4 * k + 2] & 0xFF) << 16) | ((uint32_t)(codes[4 * k + 3] & 0xFF) << 24);
                reinterpret_cast<uint4*>(dst)[0] = make_uint4(out[0], out[1], out[2], out[3]);
                reinterpret_cast<uint4*>(dst)[1] = make_uint4(out[4], out[5], out[6], out[7]);
            } else if constexpr (WBITS == 4) {
                uint32_t out[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t word = 0;
#pragma unroll
                    for (int j = 0; j < 8; ++j) word |= (uint32_t)(codes[8 * k + j] & 0xF) << (4 * j);
                    out[k] = word;
                }
                reinterpret_cast<uint4*>(dst)[0] = make_uint4(out[0], out[1], out[2], out[3]);
            } else {
                uint32_t out[2];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    uint32_t word = 0;
#pragma unroll
                    for (int j = 0; j < 16; ++j) word |= (uint32_t)(codes[16 * k + j] & 0x3) << (2 * j);
                    out[k] = word;
                }
                reinterpret_cast<uint2*>(dst)[0] = make_uint2(out[0], out[1]);
            }
        }
        __syncthreads();
    }
}

cudaError_t launch_pack_weights(const float* w, int64_t rows, int cols, int wbits, uint8_t* packed,
                                float* scales, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    const int grid = (int)(rows < 1048576 ? rows : 1048576);
    const RowsF32 src{w, cols};
    if (wbits == 8) k_pack_rows<8><<<grid, 256, 0, s>>>(src, rows, cols, packed, scales);
    else if (wbits == 4) k_pack_rows<4><<<grid, 256, 0, s>>>(src, rows, cols, packed, scales);
    else k_pack_rows<2><<<grid, 256, 0, s>>>(src, rows, cols, packed, scales);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// FP8 requantiser, one warp per row with the row's codes in registers.
//
// Lane l holds 16-code chunks l, l + 32, ... (16-byte loads, coalesced).
// The row's amax needs no decoding of most codes: for E4M3 the magnitude
// order of the non-NaN codes is the integer order of their low 7 bits, and
// within a block every value is code * the block's scale (rounding is
// monotone), so amax = max over blocks of |value(largest code) * scale|,
// exactly the maximum of |value * scale| over the row.  The codes are then
// decoded once each (E4M3 -> f16 is exact, f16 -> fp32 is exact), scaled
// by their block's scale (one fp32 multiply, as the definition), quantised
// and packed.  Rows up to kRequantMaxCols codes; NaN codes are unspecified.
// ---------------------------------------------------------------------------
constexpr int kRequantMaxChunks = 16;  // per lane: 16 x 16 codes
constexpr int kRequantMaxCols = 32 * 16 * kRequantMaxChunks;

// Two E4M3 codes (low and high byte of v) -> two fp32 values, exactly.
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t v) {
    uint32_t h2;
    asm("{\n\t.reg .b16 lo;\n\tcvt.u16.u32 lo, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(h2) : "r"(v));
    return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// Largest 7-bit magnitude field of the 16 codes of a chunk.
__device__ __forceinline__ uint32_t chunk_max_mag(uint4 w) {
    const uint32_t m = __vmaxu4(__vmaxu4(w.x & 0x7F7F7F7Fu, w.y & 0x7F7F7F7Fu), __vmaxu4(w.z & 0x7F7F7F7Fu, w.w & 0x7F7F7F7Fu));
    return max(max(m & 0xFFu, (m >> 8) & 0xFFu), max((m >> 16) & 0xFFu, m >> 24));
}

template <int WBITS, int NCH>
__global__ void __launch_bounds__(256) k_requant_fp8_rows(const uint8_t* __restrict__ w8, const float* __restrict__ bs,
                                                          int64_t rows, int cols, int block, int nbc,
                                                          uint8_t* __restrict__ packed, float* __restrict__ scales) {
    constexpr int qmax = WBITS == 8 ? 127 : WBITS == 4 ? 7 : 1;
    constexpr float qminf = -(float)(1 << (WBITS - 1));
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int nch = cols / 16;
    const uint4* src = reinterpret_cast<const uint4*>(w8 + r * cols);
    const float* bsr = bs + (r / block) * nbc;
    uint4 w[NCH];
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
        const int c = lane + 32 * j;
        w[j] = c < nch ? ld_stream_v4(src + c) : make_uint4(0, 0, 0, 0);
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
        const int c = lane + 32 * j;
        if (c < nch) {
            const float top = e4m3x2_to_f32(chunk_max_mag(w[j])).x;
            amax = fmaxf(amax, fabsf(__fmul_rn(top, __ldg(bsr + (16 * c) / block))));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    float sc = 0.0f, is = 0.0f;
    if (amax >= FLT_MIN) {
        sc = __fdiv_rn(amax, (float)qmax);
        is = __fdiv_rn(1.0f, sc);
    }
    const bool zero = !(sc > 0.0f);
    if (lane == 0) scales[r] = sc;
    uint8_t* dst = packed + r * ((int64_t)cols * WBITS / 8);
#pragma unroll
    for (int j = 0; j < NCH; ++j) {
        const int c = lane + 32 * j;
        if (c >= nch) continue;
        const float bsc = __ldg(bsr + (16 * c) / block);
        const uint32_t ww[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
        int code[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 a = e4m3x2_to_f32(ww[k] & 0xFFFFu), b = e4m3x2_to_f32(ww[k] >> 16);
            const float v[4] = {a.x, a.y, b.x, b.y};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float q = roundf(__fmul_rn(__fmul_rn(v[i], bsc), is));
                q = fminf(fmaxf(q, qminf), (float)qmax);
                code[4 * k + i] = zero ? 0 : (int)q;
            }
        }
        if constexpr (WBITS == 8) {
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                o[k] = (uint32_t)(code[4 * k] & 0xFF) | ((uint32_t)(code[4 * k + 1] & 0xFF) << 8) |
                       ((uint32_t)(code[4 * k + 2] & 0xFF) << 16) | ((uint32_t)(code[4 * k + 3] & 0xFF) << 24);
            reinterpret_cast<uint4*>(dst)[c] = make_uint4(o[0], o[1], o[2], o[3]);
        } else if constexpr (WBITS == 4) {
            uint32_t o[2] = {0u, 0u};
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i >> 3] |= (uint32_t)(code[i] & 0xF) << (4 * (i & 7));
            reinterpret_cast<uint2*>(dst)[c] = make_uint2(o[0], o[1]);
        } else {
            uint32_t o = 0u;
#pragma unroll
            for (int i = 0; i < 16; ++i) o |= (uint32_t)(code[i] & 0x3) << (2 * i);
            reinterpret_cast<uint32_t*>(dst)[c] = o;
        }
    }
}

template <int WBITS>
static cudaError_t launch_requant_rows(const uint8_t* w8, const float* bs, int64_t rows, int cols, int block,
                                       uint8_t* packed, float* scales, cudaStream_t s) {
    const int nbc = (cols + block - 1) / block;
    const int64_t grid = (rows + 7) / 8;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const int per_lane = (cols / 16 + 31) / 32;
    if (per_lane <= 4)
        k_requant_fp8_rows<WBITS, 4><<<(unsigned)grid, 256, 0, s>>>(w8, bs, rows, cols, block, nbc, packed, scales);
    else if (per_lane <= 8)
        k_requant_fp8_rows<WBITS, 8><<<(unsigned)grid, 256, 0, s>>>(w8, bs, rows, cols, block, nbc, packed, scales);
    else if (per_lane <= 12)
        k_requant_fp8_rows<WBITS, 12><<<(unsigned)grid, 256, 0, s>>>(w8, bs, rows, cols, block, nbc, packed, scales);
    else
        k_requant_fp8_rows<WBITS, 16><<<(unsigned)grid, 256, 0, s>>>(w8, bs, rows, cols, block, nbc, packed, scales);
    return cudaGetLastError();
}

cudaError_t launch_requant_fp8(const uint8_t* w8, const float* block_scales, int64_t rows, int cols, int block,
                               int wbits, uint8_t* packed, float* scales, cudaStream_t s) {
    if (rows == 0) return cudaSuccess;
    // the warp-per-row kernel: 16-byte aligned rows of at most kRequantMaxCols codes
    if (cols <= kRequantMaxCols && cols % 16 == 0 && reinterpret_cast<uintptr_t>(w8) % 16 == 0 &&
        (int64_t)cols * wbits / 8 % 4 == 0) {
        if (wbits == 8) return launch_requant_rows<8>(w8, block_scales, rows, cols, block, packed, scales, s);
        if (wbits == 4) return launch_requant_rows<4>(w8, block_scales, rows, cols, block, packed, scales, s);
        return launch_requant_rows<2>(w8, block_scales, rows, cols, block, packed, scales, s);
    }
    const int grid = (int)(rows < 1048576 ? rows : 1048576);
    const RowsFp8Block src{w8, block_scales, cols, block, (cols + block - 1) / block};
    if (wbits == 8) k_pack_rows<8><<<grid, 256, 0, s>>>(src, rows, cols, packed, scales);
    else if (wbits == 4) k_pack_rows<4><<<grid, 256, 0, s>>>(src, rows, cols, packed, scales);
    else k_pack_rows<2><<<grid, 256, 0, s>>>(src, rows, cols, packed, scales);
    return cudaGetLastError();
}

}  // namespace moe
