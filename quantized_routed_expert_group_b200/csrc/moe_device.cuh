// moe_device.cuh -- device helpers shared by the MoE layer kernels (sm_100a).
//
// The arithmetic here is the integer-dot form of the colibri engine's expert
// matmuls (GeekNews "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", §구현된 주요 기능:
// Q8_0-style int8 activations times int8 / packed int4 weights with per-row
// scales, dequantised on use), restated for CUDA cores: __dp4a on four int8
// lanes instead of AVX2 maddubs.
#pragma once

#include <cfloat>
#include <cstdint>
#include <cuda_runtime.h>

namespace moe {

constexpr int kQBlock = 32;           // Q8_0 block length
constexpr unsigned kFull = 0xffffffffu;

// Error codes written to the workspace error word.
constexpr int kErrIndex = 1;
constexpr int kErrTimeout = 2;
constexpr int kErrWorkspace = 3;  // the fused path's control region is not initialised

__device__ __forceinline__ void set_error(int32_t* err, int code) {
    if (err) atomicCAS(reinterpret_cast<int*>(err), 0, code);
}

// 128-bit read-only streaming load: weights are read once per call, so they
// bypass L1 and ask L2 for 256-byte sector prefetch.
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p));
    return r;
}

__device__ __forceinline__ uint2 ld_stream_v2(const void* p) {
    uint2 r;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ float4 ld_stream_f4(const float4* p) {
    float4 r;
    asm("ld.global.nc.L1::no_allocate.L2::256B.v4.f32 {%0, %1, %2, %3}, [%4];"
        : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
        : "l"(p));
    return r;
}

// 128-bit read-only load that may stay in L1 (activations, reused across rows).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

// Activation block of 32 int8 codes, kept in the order the weight format wants:
// for int8 weights the natural order (8 words of 4 codes), for int4 weights the
// even and odd elements of each group of 8 split apart, matching the low and
// high nibbles of one packed 32-bit weight word, for int2 weights the elements
// of each half block (16) grouped by their 2-bit field position m.
struct ActBlock {
    uint32_t v[8];
};

__device__ __forceinline__ ActBlock act_natural(uint4 lo, uint4 hi) {
    ActBlock a;
    a.v[0] = lo.x; a.v[1] = lo.y; a.v[2] = lo.z; a.v[3] = lo.w;
    a.v[4] = hi.x; a.v[5] = hi.y; a.v[6] = hi.z; a.v[7] = hi.w;
    return a;
}

// Natural -> nibble order: word pair (x[8k..8k+3], x[8k+4..8k+7]) becomes
// (x[8k], x[8k+2], x[8k+4], x[8k+6]) and (x[8k+1], x[8k+3], x[8k+5], x[8k+7]).
__device__ __forceinline__ ActBlock act_nibble_order(uint4 lo, uint4 hi) {
    const uint32_t n[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    ActBlock a;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        a.v[2 * k] = __byte_perm(n[2 * k], n[2 * k + 1], 0x6420);
        a.v[2 * k + 1] = __byte_perm(n[2 * k], n[2 * k + 1], 0x7531);
    }
    return a;
}

// Natural -> crumb order: for each half block h (elements 16h..16h+15, four
// natural words n[4h..4h+3]) word 4h + m holds elements 16h + 4j + m, j = 0..3
// (a 4 x 4 byte transpose), matching field m of the 4 bytes of one packed-int2
// weight word.
__device__ __forceinline__ ActBlock act_crumb_order(uint4 lo, uint4 hi) {
    const uint32_t n[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    ActBlock a;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const uint32_t t0 = __byte_perm(n[4 * h], n[4 * h + 1], 0x5140);      // b0 b0' b1 b1'
        const uint32_t t1 = __byte_perm(n[4 * h + 2], n[4 * h + 3], 0x5140);
        const uint32_t u0 = __byte_perm(n[4 * h], n[4 * h + 1], 0x7362);      // b2 b2' b3 b3'
        const uint32_t u1 = __byte_perm(n[4 * h + 2], n[4 * h + 3], 0x7362);
        a.v[4 * h + 0] = __byte_perm(t0, t1, 0x5410);
        a.v[4 * h + 1] = __byte_perm(t0, t1, 0x7632);
        a.v[4 * h + 2] = __byte_perm(u0, u1, 0x5410);
        a.v[4 * h + 3] = __byte_perm(u0, u1, 0x7632);
    }
    return a;
}

// 64 * the exact dot of one packed-int2 block (8 bytes = 32 codes, element
// 4j + m in bits 2m..2m+1 of byte j) with a crumb-ordered activation block:
// shifting field m to the top two bits of its byte makes the byte 64 * code as
// a signed int8, so each field position is one dp4a; |64 * dot| <= 520192.
__device__ __forceinline__ int dot_block_i2_x64(uint32_t w0, uint32_t w1, const ActBlock& a) {
    int acc = 0;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        acc = __dp4a(static_cast<int>((w0 << (6 - 2 * m)) & 0xC0C0C0C0u), static_cast<int>(a.v[m]), acc);
        acc = __dp4a(static_cast<int>((w1 << (6 - 2 * m)) & 0xC0C0C0C0u), static_cast<int>(a.v[4 + m]), acc);
    }
    return acc;
}

// Exact int32 dot of one packed-int4 block (16 bytes = 32 codes, element 2j in
// the low nibble of byte j) with a nibble-ordered activation block.  Each
// nibble is moved to the top of its byte, which makes the byte 16 * code as a
// signed int8; the sum is therefore 16 * dot and the final shift is exact.
__device__ __forceinline__ int dot_block_i4(uint4 w, const ActBlock& a) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    int acc = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int lo16 = static_cast<int>((ww[k] << 4) & 0xF0F0F0F0u);
        const int hi16 = static_cast<int>(ww[k] & 0xF0F0F0F0u);
        acc = __dp4a(lo16, static_cast<int>(a.v[2 * k]), acc);
        acc = __dp4a(hi16, static_cast<int>(a.v[2 * k + 1]), acc);
    }
    return acc >> 4;
}

// dp4a with an unsigned first operand (four u8) and a signed second (four s8).
__device__ __forceinline__ int dp4a_us(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// (a & b) ^ c in one logic op.
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// -128 * (sum of the 16 activation codes that meet low nibbles: words 0, 2,
// 4, 6 of a nibble-ordered block); the starting value of dot_block_i4_x16.
__device__ __forceinline__ int act_lo_corr(const ActBlock& a) {
    int s = __dp4a(static_cast<int>(a.v[0]), 0x01010101, 0);
    s = __dp4a(static_cast<int>(a.v[2]), 0x01010101, s);
    s = __dp4a(static_cast<int>(a.v[4]), 0x01010101, s);
    s = __dp4a(static_cast<int>(a.v[6]), 0x01010101, s);
    return -128 * s;
}

// 16 * the exact dot of a packed-int4 block with a nibble-ordered activation
// block, in fewer operations than dot_block_i4: the low nibbles are read in
// excess-8 form ((w & 0x0F0F0F0F) ^ 0x08080808 = code + 8 as an unsigned
// byte, one logic op) and the excess is removed by starting the high-nibble
// sum at corr = act_lo_corr(a); the high nibbles stay 16 * code.
__device__ __forceinline__ int dot_block_i4_x16(uint4 w, const ActBlock& a, int corr) {
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    int lo = 0, hi = corr;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        lo = dp4a_us(and_xor(ww[k], 0x0F0F0F0Fu, 0x08080808u), a.v[2 * k], lo);
        hi = __dp4a(static_cast<int>(ww[k] & 0xF0F0F0F0u), static_cast<int>(a.v[2 * k + 1]), hi);
    }
    return 16 * lo + hi;
}

// Exact int32 dot of one int8 block (32 bytes) with a natural-order block.
__device__ __forceinline__ int dot_block_i8(uint4 w0, uint4 w1, const ActBlock& a) {
    int acc = 0;
    acc = __dp4a(static_cast<int>(w0.x), static_cast<int>(a.v[0]), acc);
    acc = __dp4a(static_cast<int>(w0.y), static_cast<int>(a.v[1]), acc);
    acc = __dp4a(static_cast<int>(w0.z), static_cast<int>(a.v[2]), acc);
    acc = __dp4a(static_cast<int>(w0.w), static_cast<int>(a.v[3]), acc);
    acc = __dp4a(static_cast<int>(w1.x), static_cast<int>(a.v[4]), acc);
    acc = __dp4a(static_cast<int>(w1.y), static_cast<int>(a.v[5]), acc);
    acc = __dp4a(static_cast<int>(w1.z), static_cast<int>(a.v[6]), acc);
    acc = __dp4a(static_cast<int>(w1.w), static_cast<int>(a.v[7]), acc);
    return acc;
}

template <int WBITS>
__device__ __forceinline__ ActBlock load_act_block(const int8_t* q) {
    const uint4 lo = ld_nc_v4(q);
    const uint4 hi = ld_nc_v4(q + 16);
    if constexpr (WBITS == 4) return act_nibble_order(lo, hi);
    else if constexpr (WBITS == 2) return act_crumb_order(lo, hi);
    else return act_natural(lo, hi);
}

// One weight block of a row: 32 codes = 8 bytes (int2, in a.x, a.y), 16 bytes
// (int4) or 32 bytes (int8).
template <int WBITS>
struct WBlock {
    uint4 a, b;
};

template <int WBITS>
__device__ __forceinline__ WBlock<WBITS> load_w_block(const uint8_t* row, int blk) {
    WBlock<WBITS> w;
    if constexpr (WBITS == 4) {
        w.a = ld_stream_v4(row + 16 * blk);
        w.b = make_uint4(0, 0, 0, 0);
    } else if constexpr (WBITS == 2) {
        const uint2 v = ld_stream_v2(row + 8 * blk);
        w.a = make_uint4(v.x, v.y, 0, 0);
        w.b = make_uint4(0, 0, 0, 0);
    } else {
        w.a = ld_stream_v4(row + 32 * blk);
        w.b = ld_stream_v4(row + 32 * blk + 16);
    }
    return w;
}

template <int WBITS>
__device__ __forceinline__ int dot_block(const WBlock<WBITS>& w, const ActBlock& a) {
    if constexpr (WBITS == 4) return dot_block_i4(w.a, a);
    else if constexpr (WBITS == 2) return dot_block_i2_x64(w.a.x, w.a.y, a) >> 6;
    else return dot_block_i8(w.a, w.b, a);
}

// The block dot times the factor dot_scale<WBITS>() (64 for int2, 16 for
// int4, 1 for int8) as an exact integer (below 2^24, so exact as a float too);
// corr is act_corr<WBITS>(a).
template <int WBITS>
__device__ __forceinline__ int dot_block_scaled(const WBlock<WBITS>& w, const ActBlock& a, int corr) {
    if constexpr (WBITS == 4) return dot_block_i4_x16(w.a, a, corr);
    else if constexpr (WBITS == 2) return dot_block_i2_x64(w.a.x, w.a.y, a);
    else return dot_block_i8(w.a, w.b, a);
}

// 1 / that factor (a power of two: scaling by it is exact).
template <int WBITS>
__device__ __forceinline__ float dot_unscale() {
    return WBITS == 4 ? 0.0625f : WBITS == 2 ? 0.015625f : 1.0f;
}

template <int WBITS>
__device__ __forceinline__ int act_corr(const ActBlock& a) {
    if constexpr (WBITS == 4) return act_lo_corr(a);
    else return 0;
}

// Q8_0 of one block held one value per lane: d = amax/127 (IEEE divide),
// q = round-half-away(v * (1/d)) clamped to [-127, 127]; amax < FLT_MIN
// gives d = 0, q = 0.  Every lane of the warp must call it.
__device__ __forceinline__ void q8_0_warp(float v, int8_t& q, float& d) {
    float a = fabsf(v);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
    if (!(a >= FLT_MIN)) {
        d = 0.0f;
        q = 0;
        return;
    }
    d = __fdiv_rn(a, 127.0f);
    const float id = __fdiv_rn(1.0f, d);
    float r = roundf(__fmul_rn(v, id));
    r = fminf(fmaxf(r, -127.0f), 127.0f);
    q = static_cast<int8_t>(static_cast<int>(r));
}

// Butterfly reduction of V per-lane values across the warp (V a power of two,
// 1 <= V <= 32): afterwards every lane holds the full sum of value index
// (lane >> (5 - log2 V)).  Costs V - 1 + (5 - log2 V) shuffles instead of
// 5 V for V independent reductions.
template <int V>
__device__ __forceinline__ float warp_reduce_many(float (&v)[V], int lane) {
    int n = V;
    int off = 16;
#pragma unroll
    for (; n > 1; n >>= 1, off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < n / 2; ++i) {
            const float send = upper ? v[i] : v[i + n / 2];
            const float keep = upper ? v[i + n / 2] : v[i];
            v[i] = keep + __shfl_xor_sync(kFull, send, off);
        }
    }
    float r = v[0];
#pragma unroll
    for (; off > 0; off >>= 1) r += __shfl_xor_sync(kFull, r, off);
    return r;
}

template <int V>
struct Log2 {
    static constexpr int value = V <= 1 ? 0 : 1 + Log2<V / 2>::value;
};
template <>
struct Log2<1> {
    static constexpr int value = 0;
};

// SwiGLU activation of one row: silu(g) * u = g / (1 + e^-g) * u, in fp32
// (accurate expf and IEEE division; no fast-math).
__device__ __forceinline__ float silu_mul(float g, float u) {
    return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.0f, expf(-g))), u);
}

// Compensated ("double-float") dot-product accumulation in fp32.  The
// product of two fp32 values is split exactly into hi + lo with one fma
// (TwoProduct) and added into a running (sum, err) pair with TwoSum (Knuth),
// so the pair carries the running sum to about 2^-48 relative instead of
// fp32's 2^-24, using only fp32 instructions (fp64 arithmetic on CUDA cores is
// a narrow pipe on B200).  The pair is folded into fp64 at the end.
struct DFAcc {
    float hi = 0.0f, lo = 0.0f;
    __device__ __forceinline__ void add_prod(float a, float b) {
        const float p = __fmul_rn(a, b);
        const float pe = __fmaf_rn(a, b, -p);  // exact product error
        const float t = __fadd_rn(hi, p);
        const float bp = __fsub_rn(t, hi);
        const float e = __fadd_rn(__fsub_rn(hi, __fsub_rn(t, bp)), __fsub_rn(p, bp));  // exact sum error
        hi = t;
        lo = __fadd_rn(lo, __fadd_rn(e, pe));
    }
    __device__ __forceinline__ double value() const { return (double)hi + (double)lo; }
};

// Order-preserving unsigned key of a double (larger value -> larger key;
// -0.0 is folded into +0.0 so that equal values give equal keys).
__device__ __forceinline__ unsigned long long order_key(double v) {
    v = v + 0.0;
    const long long b = __double_as_longlong(v);
    return b >= 0 ? (unsigned long long)b ^ 0x8000000000000000ull : ~(unsigned long long)b;
}

// Adaptive expert top-p of one token's k <= 32 picks, by the token's warp
// (GeekNews "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", §모델 다운로드와 실행,
// option list: an adaptive expert top-p; the rule is this library's nucleus
// reading).  Lane j < k holds pick j's unbiased s (sj); ssum is the sum of all
// k picks' s in pick order.  The picks are ranked by s (larger first, ties to
// the earlier pick); the first m in rank order are kept, m the smallest count
// whose running sum of s / ssum (fp64, in rank order) reaches topp, or k.
// Returns whether lane j's pick is kept and sets *skept to the kept picks' s
// summed in pick order.  Lanes >= k get false.
__device__ __forceinline__ bool topp_keep(double sj, double ssum, int k, float topp, int lane, double* skept) {
    int rank = 0;
    for (int i = 0; i < k; ++i) {
        const double si = __shfl_sync(kFull, sj, i);
        rank += (si > sj || (si == sj && i < lane)) ? 1 : 0;
    }
    if (lane >= k) rank = 32;
    double cum = 0.0;
    int m = k;
    for (int r = 0; r < k; ++r) {  // the same values in every lane: a uniform exit
        const int who = __ffs(__ballot_sync(kFull, rank == r)) - 1;
        cum += __shfl_sync(kFull, sj, who < 0 ? 0 : who) / ssum;
        if (cum >= (double)topp) {
            m = r + 1;
            break;
        }
    }
    const bool keep = rank < m;
    double sk = 0.0;
    for (int i = 0; i < k; ++i) {
        const double si = __shfl_sync(kFull, sj, i);
        if (__shfl_sync(kFull, keep ? 1 : 0, i)) sk += si;
    }
    *skept = sk;
    return keep;
}

// Arg-max of (key, index) over the warp: larger key wins, ties to the lower index.
__device__ __forceinline__ void warp_argmax_key(unsigned long long& k, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long ok = __shfl_xor_sync(kFull, k, o);
        const int oi = __shfl_xor_sync(kFull, i, o);
        if (ok > k || (ok == k && oi < i)) {
            k = ok;
            i = oi;
        }
    }
}

// Arg-max over the warp with ties to the lower index.
__device__ __forceinline__ void warp_argmax(double& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(kFull, v, o);
        const int oi = __shfl_xor_sync(kFull, i, o);
        if (ov > v || (ov == v && oi < i)) {
            v = ov;
            i = oi;
        }
    }
}

}  // namespace moe
