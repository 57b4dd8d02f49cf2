// moe_tc.cuh -- the tensor-core building blocks of the batched expert path
// (sm_100a): tiled TMA loads, TMEM allocation, tcgen05.mma kind::i8 with its
// descriptors, TMEM loads, and the int4 / int2 -> int8 widening of packed
// weight tiles into the layout the MMA reads.
//
// The arithmetic is the integer-dot form of the colibri engine's expert
// matmuls (GeekNews "Show HN: 느린 컴퓨터에서 GLM 5.2 실행하기", §구현된 주요 기능:
// Q8_0-style int8 activations times packed int4 / int8 weights with per-row
// scales; "Batch-union MoE": each unique expert applied to every position
// routed to it).  One MMA of kind::i8 has K = 32, which is exactly one Q8_0
// block, so every MMA produces the exact int32 block dots of a 128-row weight
// tile with N tokens; the per-token block scale is applied afterwards.
//
// Shared-memory operand layout ("K-major, 128-byte swizzle"): a tile of R rows
// with 128 bytes (128 int8 codes) of K per row; row r starts at byte 128 r and
// its 16-byte chunk c is stored at chunk position c ^ (r mod 8).  The tile
// base is 1024-byte aligned (the swizzle is applied to address bits), so a
// TMA load with 128-byte swizzle and the converter's stores agree on it.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "moe_ptx.cuh"

namespace moe {
namespace tc {

constexpr int kTileRows = 128;  // weight rows per MMA (M)
constexpr int kStageK = 128;    // int8 codes of K per pipeline stage (4 Q8_0 blocks)
constexpr int kBlocksPerStage = kStageK / 32;
constexpr int kMaxN = 64;       // tokens per unit (MMA N, in steps of 16)
constexpr int kTileBytes = kTileRows * kStageK;  // one widened weight tile of a stage

// Exact digit planes of the block-scaled activations.  A token's Q8_0 block
// scales d_b = m_b 2^e_b (fp32: m_b < 2^24 an integer) share the exponent
// E = min_b e_b; with spread = max_b e_b - E <= kMaxSpread, every scaled code
// q m_b 2^(e_b - E) is an integer below 127 * 2^32 in magnitude and splits
// exactly into kPlanes signed base-256 digits, each an int8.  So
//   sum_b d_b dot_b(w, q) = 2^E sum_p 256^p (w . plane_p)
// and the tensor core accumulates each plane's product in int32 over the
// whole K (|w . plane_p| <= K * 127 * 128 < 2^31 for K <= 2^17).
constexpr int kPlanes = 5;
constexpr int kMaxSpread = 8;
constexpr int kChunk = 48;  // tokens per unit of the grouped GEMMs (kPlanes * 48 = 240 <= 256 MMA columns)
static_assert(kChunk <= 64, "the epilogue holds a chunk's tokens in two lanes each");

// Integer mantissa and exponent of a finite fp32 value v >= 0: v = m 2^e with
// m < 2^24 (m = 0 for v = 0).
__device__ __forceinline__ void f32_mant_exp(float v, uint32_t& m, int& e) {
    const uint32_t b = __float_as_uint(v);
    const uint32_t f = (b >> 23) & 0xFFu;
    m = f ? ((b & 0x7FFFFFu) | 0x800000u) : (b & 0x7FFFFFu);
    e = f ? (int)f - 150 : -149;
}

// A unit of work of the grouped GEMMs: one 128-row tile of one expert's
// weight matrix applied to a chunk of <= kChunk of the expert's tokens.
struct TcUnit {
    int prow0;  // first row of the chunk in the padded row space
    int ntok;   // tokens of the chunk (1 .. kChunk)
    int wrow0;  // first weight row in the bank's matrix (expert * rows + 128 * tile)
    int info;   // tile index | kUnitShared
};
constexpr int kUnitShared = 1 << 16;

// ---------------------------------------------------------------------------
// TMA (tiled, 2-D) and its tensor map
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Box at (x, y) of a 2-D tensor map into this CTA's shared memory, completing
// on `bar` (x: innermost coordinate, in elements).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                                 uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, "
        "%3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(pol)
        : "memory");
}

// L2 policy for tiles read by several CTAs shortly after one another.
__device__ __forceinline__ uint64_t l2_evict_last_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Make this thread's generic-proxy writes to shared memory visible to the
// async proxy (the tensor core reads operands through it).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMEM
// ---------------------------------------------------------------------------
// Allocate ncols columns (a power of two >= 32) for this CTA; one full warp
// calls it; the base address lands in *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane (the warp's lane
// quarter is fixed by its index in the warpgroup: lanes 32 (warp % 4) ..).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// MMA
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor of a K-major tile with 128-byte rows and
// 128-byte swizzle: start address >> 4 (bits 0-13), leading offset 16 B
// (unused by this layout), stride between 8-row groups 1024 B (bits 32-45),
// descriptor version 1 (bit 46), swizzle mode "128B" (bits 61-63).  Advancing
// K by 32 codes adds 2 to the start field.
__device__ __forceinline__ uint64_t desc_k128_sw128(const void* tile) {
    const uint32_t a = smem_addr(tile);
    return (uint64_t)((a >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) |
           ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::i8 with signed A and B, int32 accumulator,
// both operands K-major, M = 128 and N (a multiple of 16, <= 256).
__device__ __forceinline__ uint32_t idesc_i8(int n) {
    return (2u << 4)            // D: s32
           | (1u << 7)          // A: s8
           | (1u << 10)         // B: s8
           | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kTileRows >> 4) << 24);
}

// D[128 x N] (TMEM, int32) = A[128 x 32] . B[N x 32]^T (+ D when accumulate).
// Issued by one thread.
__device__ __forceinline__ void mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                      bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
        : "memory");
}

// Arrive once on `bar` when every MMA this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

// ---------------------------------------------------------------------------
// Widening of packed weight codes into the K-major 128-byte-swizzle layout
// ---------------------------------------------------------------------------
// Byte offset of 16-byte chunk c (0..7) of row r in a swizzled tile.
__device__ __forceinline__ uint32_t sw128_chunk(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// Four packed int4 bytes (codes 8i .. 8i+7: element 2j in the low nibble of
// byte j) -> eight int8 codes in element order (two words).  A nibble is
// sign-extended by OR-ing 0xF0 into its byte when its bit 3 is set; the
// per-byte mask times 0x1E is exactly that 0xF0 (no carries between bytes).
__device__ __forceinline__ void widen_i4x8(uint32_t w, uint32_t& o0, uint32_t& o1) {
    const uint32_t lo = w & 0x0F0F0F0Fu;
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
    const uint32_t slo = lo | ((lo & 0x08080808u) * 0x1Eu);
    const uint32_t shi = hi | ((hi & 0x08080808u) * 0x1Eu);
    o0 = __byte_perm(slo, shi, 0x5140);  // e0 e1 e2 e3
    o1 = __byte_perm(slo, shi, 0x7362);  // e4 e5 e6 e7
}

// One packed int2 byte quad (codes 16i .. 16i+15: element 4j + m in bits
// 2m..2m+1 of byte j) -> sixteen int8 codes in element order (four words).
__device__ __forceinline__ void widen_i2x16(uint32_t w, uint32_t (&o)[4]) {
    uint32_t f[4];  // f[m]: field m of bytes 0..3, sign-extended (codes 4j + m)
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const uint32_t v = (w >> (2 * m)) & 0x03030303u;
        f[m] = v | ((v & 0x02020202u) * 0x7Eu);  // bit 1 set: OR 0xFC into the byte (0x02 * 0x7E = 0xFC)
    }
    // byte j of the output block = element 4j' + m: transpose the 4 x 4 bytes
    const uint32_t t0 = __byte_perm(f[0], f[1], 0x5140);  // e0 e1 e4 e5
    const uint32_t t1 = __byte_perm(f[2], f[3], 0x5140);  // e2 e3 e6 e7
    const uint32_t u0 = __byte_perm(f[0], f[1], 0x7362);  // e8 e9 e12 e13
    const uint32_t u1 = __byte_perm(f[2], f[3], 0x7362);  // e10 e11 e14 e15
    o[0] = __byte_perm(t0, t1, 0x5410);  // e0 e1 e2 e3
    o[1] = __byte_perm(t0, t1, 0x7632);  // e4 e5 e6 e7
    o[2] = __byte_perm(u0, u1, 0x5410);  // e8 .. e11
    o[3] = __byte_perm(u0, u1, 0x7632);  // e12 .. e15
}

// Widen row r of a packed staging tile into row r of a swizzled int8 tile.
// int4 staging rows are 64 bytes loaded with 64-byte swizzle (chunk c of row
// r at chunk position c ^ ((r >> 1) & 3)); int2 staging rows are 32 bytes
// loaded with 32-byte swizzle (chunk c at c ^ ((r >> 2) & 1)).
template <int WBITS>
__device__ __forceinline__ void widen_row(const uint8_t* raw, uint8_t* tile, int r) {
    if constexpr (WBITS == 4) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 w = *reinterpret_cast<const uint4*>(raw + r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
            uint4 a, b;
            widen_i4x8(w.x, a.x, a.y);
            widen_i4x8(w.y, a.z, a.w);
            widen_i4x8(w.z, b.x, b.y);
            widen_i4x8(w.w, b.z, b.w);
            *reinterpret_cast<uint4*>(tile + sw128_chunk(r, 2 * c)) = a;
            *reinterpret_cast<uint4*>(tile + sw128_chunk(r, 2 * c + 1)) = b;
        }
    } else if constexpr (WBITS == 2) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint4 w = *reinterpret_cast<const uint4*>(raw + r * 32 + ((c ^ ((r >> 2) & 1)) << 4));
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t o[4];
                widen_i2x16(ww[q], o);
                *reinterpret_cast<uint4*>(tile + sw128_chunk(r, 4 * c + q)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
        }
    }
}

// The digit-plane GEMM's widening: each packed code moved to the top of its
// byte, i.e. 2^(8 - WBITS) * code as an int8 (16 code for int4, 64 code for
// int2; int8 rows are not widened), so that only shifts, masks and byte
// permutes are needed; the GEMM's epilogue removes the power of two exactly
// (kWidenShift).  Same output layout as widen_row.
template <int WBITS>
constexpr int kWidenShift = WBITS == 4 ? 4 : WBITS == 2 ? 6 : 0;

// One 16-byte chunk c of packed row r (32 int4 or 64 int2 codes), held in
// registers -> its 32 or 64 widened bytes of the SW128 tile.
template <int WBITS>
__device__ __forceinline__ void widen_chunk_regs_top(const uint4 w, uint8_t* tile, int r, int c) {
    if constexpr (WBITS == 4) {
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        uint32_t o[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t ev = (ww[q] << 4) & 0xF0F0F0F0u;  // elements 0, 2, 4, 6 of the word: 16 code
            const uint32_t od = ww[q] & 0xF0F0F0F0u;         // elements 1, 3, 5, 7
            o[2 * q] = __byte_perm(ev, od, 0x5140);
            o[2 * q + 1] = __byte_perm(ev, od, 0x7362);
        }
        *reinterpret_cast<uint4*>(tile + sw128_chunk(r, 2 * c)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(tile + sw128_chunk(r, 2 * c + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
    } else if constexpr (WBITS == 2) {
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t f[4];  // f[m]: field m of bytes 0..3 at the top of its byte (64 code of element 4j + m)
#pragma unroll
            for (int m = 0; m < 4; ++m) f[m] = (ww[q] << (6 - 2 * m)) & 0xC0C0C0C0u;
            const uint32_t t0 = __byte_perm(f[0], f[1], 0x5140);
            const uint32_t t1 = __byte_perm(f[2], f[3], 0x5140);
            const uint32_t u0 = __byte_perm(f[0], f[1], 0x7362);
            const uint32_t u1 = __byte_perm(f[2], f[3], 0x7362);
            *reinterpret_cast<uint4*>(tile + sw128_chunk(r, 4 * c + q)) =
                make_uint4(__byte_perm(t0, t1, 0x5410), __byte_perm(t0, t1, 0x7632), __byte_perm(u0, u1, 0x5410),
                           __byte_perm(u0, u1, 0x7632));
        }
    }
}

// The same from a packed staging row in shared memory, TMA-loaded with the
// 64-byte (int4) or 32-byte (int2) swizzle, so that eight consecutive rows
// read eight distinct bank groups.
template <int WBITS>
__device__ __forceinline__ void widen_chunk_top(const uint8_t* raw, uint8_t* tile, int r, int c) {
    const uint4 w = WBITS == 4 ? *reinterpret_cast<const uint4*>(raw + r * 64 + ((c ^ ((r >> 1) & 3)) << 4))
                               : *reinterpret_cast<const uint4*>(raw + r * 32 + ((c ^ ((r >> 2) & 1)) << 4));
    widen_chunk_regs_top<WBITS>(w, tile, r, c);
}

// 16-byte chunks of one packed staging row.
template <int WBITS>
constexpr int raw_row_chunks() {
    return kStageK * WBITS / 8 / 16;
}

// Part `part` of `PARTS` of packed row r: its raw_row_chunks / PARTS chunks.
template <int WBITS, int PARTS>
__device__ __forceinline__ void widen_row_top(const uint8_t* raw, uint8_t* tile, int r, int part) {
    constexpr int kPer = raw_row_chunks<WBITS>() / PARTS;
    static_assert(kPer * PARTS == raw_row_chunks<WBITS>(), "row parts of whole chunks");
#pragma unroll
    for (int c = 0; c < kPer; ++c) widen_chunk_top<WBITS>(raw, tile, r, part * kPer + c);
}

// Bytes of one packed staging row of a stage (kStageK codes).
template <int WBITS>
constexpr int raw_row_bytes() {
    return kStageK * WBITS / 8;
}

// Exact float of an int32 block dot |v| < 2^22: placed in the mantissa of
// 1.5 * 2^23 and the bias subtracted (exact: same binade, integer result).
__device__ __forceinline__ float exact_i2f(uint32_t v) {
    return __fsub_rn(__int_as_float((int)(v + 0x4B400000u)), 12582912.0f);
}

}  // namespace tc
}  // namespace moe
