// moe_small.cu -- the whole MoE layer forward for small batches (T <= 4:
// decode and speculative verify) as one persistent kernel with a static
// schedule.
//
// What it computes is the layer of moe_api.cu (router, batch-union bucketing,
// SwiGLU experts on Q8_0 activations, combine; GeekNews "Show HN: 느린 컴퓨터에서
// GLM 5.2 실행하기", §구현된 주요 기능; wpnews.pro "Colibri — รัน GLM-5.2 ...",
// spec and kernel tables, "Batch-Union MoE").  How it is scheduled is B200's:
//
// * At one to four tokens the layer is a stream of ~170-400 MB of expert
//   weights, so the goal is to keep HBM busy from the first cycle to the
//   last.  Each CTA (one per SM) has a producer warp that streams the CTA's
//   share of the weights with bulk asynchronous copies (cp.async.bulk, the
//   1-D TMA form) into a ring of 48 KB shared-memory slots, and eight
//   consumer warps that do the integer dots on __dp4a.
// * The schedule is static except for the routed gate/up units at T > 1:
//   - router: CTA c computes the logits of experts 2c and 2c+1;
//   - selection: every CTA routes all tokens itself from the published
//     logits (identical decisions everywhere), so the routing costs one
//     grid-wide wait and no broadcast;
//   - gate/up: cut into units of 32 rows of one expert (one Q8_0 block of h);
//     the shared expert's unit c belongs to CTA c (it needs no routing); at
//     one token the routed experts' units continue the round robin (unit u
//     to CTA u mod grid), at more tokens they are taken from a global counter
//     (one atomic per unit), so that SMs with more bandwidth take more; the CTA
//     finishes its units: SwiGLU, Q8_0 of the 32 h values, published with
//     one release counter per expert;
//   - down + combine: CTA c owns output rows [H c / grid, H (c+1) / grid) of
//     every expert and combines them itself at the end, so no partial output
//     crosses CTAs: no float atomics, bit-reproducible results.
// * The only waits: the selection waits for every CTA's router logits (one
//   grid-wide barrier), and each down chunk waits for its expert's h (the
//   producer polls, then copies the h codes into the slot with the
//   weights).  Every wait is bounded and records a timeout in the error word.
// * Weights known before the routing (the shared expert's) are issued at the
//   kernel's first instruction, and the CTA's shared-expert down rows are
//   prefetched into L2 while the routing is computed.
// * One launch: the consumer warps quantise x and compute the CTA's router
//   logits themselves, so the weights start to stream as the kernel starts.
//   The control words it shares between CTAs are never reset (see
//   kFcMarker): each CTA reads their values before its router arrival and
//   counts from there.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>

#include "moe_device.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

// Build option of the one-token schedule (a tuning knob; the default is the
// measured best): consumer groups.
#ifndef MOE_SMALL_GROUPS
#define MOE_SMALL_GROUPS 2
#endif

constexpr int kConsumerWarps = 8;  // warps of one consumer group
constexpr int kConsumers = kConsumerWarps * 32;
// Warp roles: kGroups groups of consumer warps (two at one token, where the
// consumers' latency sets the pace: the groups work on alternate ring slots),
// then the producer warp (streams the items) and the finisher warp (finishes
// gate/up units).
template <int TM>
struct Roles {
    static constexpr int kGroups = TM == 1 ? MOE_SMALL_GROUPS : 1;
    static constexpr int kProducerWarp = kGroups * kConsumerWarps;
    static constexpr int kFinisherWarp = kProducerWarp + 1;
    static constexpr int kThreads = (kFinisherWarp + 1) * 32;
};
constexpr int kSlotWeightBytes = 48 * 1024;
constexpr int kMaxSlots = 4;
constexpr int kUnit = 32;          // gate/up rows per unit: one Q8_0 block of h
constexpr int kMaxOwnedRows = 64;  // output rows one CTA owns
constexpr int kScaleWin = 160;     // 16-byte aligned window over <= 32 fp32 scales
constexpr int kMaxEntryWords = 5;  // ready bitmask words (entries <= 160)
constexpr int kRouterRound = 4;    // router rows a CTA computes at a time
constexpr int kMaxKeptFast = 4;    // kept groups of the groups-of-32 selection
constexpr double kDownCost = 1.5;  // one token: time of a down byte over a gate/up byte (see owned_rows)
constexpr double kSharedUnitCost = 0.0;  // one token: a shared-expert gate/up unit against a routed one (measured: free)
constexpr int kOwnTab = 34;              // entry counts the down-row split is tabled for (top_k <= 33)
constexpr uint64_t kFcMarkerValue = 0x3130646573756646ull;
// Thread layout of the gate/up and down chunks: the 64 threads of a warp
// pair (w, w+1) split the columns (K blocks c, c + 64, ...), the 4 warp pairs
// split the rows.  Each thread loads its activation blocks once per chunk and
// reuses them for all its rows; its dots are independent chains.  A row's
// sum is the two warps' butterfly sums, added half 0 + half 1.
constexpr int kColThreads = 64;
constexpr int kRowGroups = 4;  // = consumer warps / 2
constexpr int kRowBatch = 4;       // rows reduced together
constexpr int kMaxGuBlocks = 3;    // hidden / 32 <= 192 blocks over 64 column threads
constexpr int kMaxDownBlocks = 8;  // inter / 32 <= 512

// Bounds of every wait, in nanoseconds of the global timer (legitimate waits
// last microseconds).  The producer's waits (a free ring slot, another CTA's
// h codes) give up after wait_ns (kWaitNs unless a test shortens it) and end
// the CTA's schedule with a DONE marker; every other wait (consumers on their
// producer, the producer on the consumers' routing, the finisher on the
// consumers) spans at most one producer wait plus that hand-over, so its
// bound is kSlackWaits times as long.  A wait that runs out records
// kErrTimeout in the error word; the kernel then returns.
constexpr uint64_t kWaitNs = 25ull * 1000 * 1000;
constexpr uint64_t kSlackWaits = 4;

enum ItemKind : int {
    kItemSelect = 2,
    kItemGateUp = 3,
    kItemDown = 4,
    kItemCombine = 5,
    kItemDone = 6,
    kItemSync = 7  // two groups: the other group's down outputs are complete
};

// Control region of the fused path (int32 words at a fixed workspace offset,
// the only workspace state kept from one call to the next):
//   [0, 1]  a 64-bit marker that moe_workspace_init writes; a call that does
//           not find it records kErrWorkspace and computes nothing;
//   [2]     the router barrier: each CTA adds 1, CTA 0 adds 2^31 - (grid - 1),
//           so that bit 31 flips when the last CTA arrives and the low 31
//           bits are zero again (zero after the initialisation);
//   [3]     routed gate/up units taken (T > 1);
//   [4 + e] (unit, token) pairs of entry e whose h codes are published.
// The counters are never reset: every CTA reads them before its router
// arrival, and nobody adds to them before the barrier completes, so every
// CTA counts from the same values (differences modulo 2^32).
enum : int { kFcMarker = 0, kFcBarrier = 2, kFcUnits = 3, kFcDone = 4 };

// One expert of the batch union: entry 0 is the shared expert, entry 1 + a
// the a-th routed expert in ascending id order.
struct EntryInfo {
    int expert;  // routed expert id, -1 for the shared expert
    int slot0;   // first h / y slot (bucketed position)
    int n;       // tokens
    int tok[4];
    int pad;
};

// A gate/up unit handed from the consumer warps to the finisher warp.
struct UnitRec {
    int entry;  // < 0: no more units
    int blk;
    int slot0;
    int n;
};

struct SmallGeom {
    int grid;
    int tmax;
    int nent;      // 1 + max routed entries
    int rg;        // gate/up row pairs per chunk
    int cpu;       // chunks per unit
    int nu;        // units per expert
    int rpc;       // max output rows a CTA owns
    int rd;        // down rows per chunk
    int nys;       // output slots (T*k routed + T shared)
    int nslot;
    int a_hd;  // act-area offset of the h-scale window (down chunks)
    int a_sd;  // act-area offset of the row-scale window (down chunks)
    int act_bytes;
    int slot_bytes;
    int o_xq, o_xd, o_bar, o_meta, o_urec, o_gpart, o_usc, o_ent, o_selw, o_inv, o_ys, o_misc, o_base, o_part, o_bias;
    int smem_bytes;
};

struct SmallParams {
    int T, H, I, E, G, tg, k, ns, wbits;
    float rsf;
    float topp;  // adaptive expert top-p; outside (0, 1): keep every pick
    int ep_lo, ep_hi;  // routed experts this call computes (expert parallelism): [ep_lo, ep_hi)
    const float* x;
    const float* router_w;
    const float* bias;
    moe_experts routed;
    moe_experts shared;
    int8_t* xq;
    float* xd;
    double* logits;  // [T][E] router scores s = sigmoid(logit), one row per expert from its CTA
    int32_t* idx;
    float* w;
    int32_t* counts;
    int32_t* offsets;
    int32_t* perm;
    int32_t* inv_perm;
    int32_t* active;
    int8_t* hq;
    float* hd;
    float* y;
    float* out;
    int* ctrl;  // the control region (kFc*)
    int32_t* err;
    uint64_t wait_ns;  // bound of the producer's waits (see kWaitNs)
    int fault_entry;   // test hook: the entry whose first unit's h codes are never published (-1: none)
    int rows_bulk;     // the router matrix is 16-byte aligned: router rows by bulk copy
    SmallGeom g;
    // one token: the down-row split's common finish time for each entry
    // count (see owned_rows), computed on the host
    double own_tt[kOwnTab];
};

struct SlotMeta {
    int kind;
    int entry;   // 0 shared, 1 + a routed
    int expert;  // routed expert id; -1 shared; first expert for router items
    int row0;    // first weight row of the chunk (combine: first output row)
    int nrows;
    int n;       // tokens of the entry
    int slot0;   // first h / y slot of the entry
    int blk;     // gate/up: unit block (h block index); down: row offset inside the CTA's rows
    int last;    // gate/up: last chunk of its unit
    int off_a;   // byte offset in the slot: gate scales / h scales
    int off_b;   // byte offset in the slot: up scales / down row scales
    int uc;      // gate/up: the unit's ordinal in this CTA; DONE: the CTA's unit count
    int tok[4];
};

// ---------------------------------------------------------------------------
// Geometry
// ---------------------------------------------------------------------------
static int round_up(int v, int a) { return (v + a - 1) / a * a; }

SmallGeom small_geometry(const moe_config& c, int T, int grid) {
    SmallGeom g{};
    const int H = c.hidden, I = c.inter, E = c.n_experts;
    const int rowH = H * c.wbits / 8, rowI = I * c.wbits / 8;
    g.grid = grid;
    g.tmax = T <= 1 ? 1 : T <= 2 ? 2 : 4;
    g.nent = 1 + (E < T * c.top_k ? E : T * c.top_k);
    int rg = kSlotWeightBytes / (2 * rowH);
    rg = rg > kUnit ? kUnit : rg;
    int p2 = 1;
    while (p2 * 2 <= rg) p2 *= 2;
    g.rg = rg >= 1 ? p2 : 0;
    g.cpu = g.rg > 0 ? kUnit / g.rg : 0;
    g.nu = I / kUnit;
    g.rpc = (H + grid - 1) / grid;
    // one token: the rows are split so that every CTA streams the same bytes
    // (see owned_rows), up to twice the even share
    if (g.tmax == 1) g.rpc = min(2 * g.rpc, kMaxOwnedRows);
    const int rd = kSlotWeightBytes / rowI;
    g.rd = rd > kMaxOwnedRows ? kMaxOwnedRows : rd;
    g.nys = T * c.top_k + T * c.n_shared;
    g.nslot = kMaxSlots;
    const int nbI = I / 32;
    g.a_hd = round_up(g.tmax * I, 16);
    g.a_sd = g.a_hd + round_up(g.tmax * nbI * 4 + 32, 16);
    g.act_bytes = round_up(g.a_sd + kMaxOwnedRows * 4 + 32, 128);
    if (g.act_bytes < 2 * kScaleWin) g.act_bytes = round_up(2 * kScaleWin, 128);
    g.slot_bytes = kSlotWeightBytes + g.act_bytes;
    int o = 0;
    g.o_xq = o;
    o += round_up(g.tmax * H, 128);
    g.o_xd = o;
    o += round_up(g.tmax * (H / 32) * 4, 128);
    g.o_bar = o;
    o += 256;  // full[4], empty[4], routing, ufull[2], ufree[2], gsync, gexit, rowsin, ctrl
    g.o_meta = o;
    o += round_up((int)sizeof(SlotMeta) * kMaxSlots, 128);
    g.o_urec = o;
    o += 128;  // UnitRec[2]
    g.o_gpart = o;
    o += 2 * kUnit * 2 * 8 * 4;  // [buffer][pair][half][gate/up][token]
    g.o_usc = o;
    o += 2 * kUnit * 2 * 4;  // [buffer][pair][gate/up] row scales
    g.o_ent = o;
    o += round_up(g.nent * (int)sizeof(EntryInfo), 128);
    g.o_selw = o;
    o += round_up(T * c.top_k * 4, 128);
    g.o_inv = o;
    o += round_up(T * c.top_k * 4, 128);
    g.o_ys = o;
    o += round_up(g.nys * g.rpc * 8, 128);
    g.o_misc = o;
    o += 128;
    g.o_base = o;  // the control counters at the CTA's start: [units, done[nent]]
    o += round_up((1 + g.nent) * 4, 128);
    g.o_part = o;  // router logits: [expert of the round][eighth][token] fp64
    o += kRouterRound * 8 * 4 * 8;
    g.o_bias = o;  // router correction bias [E]
    o += round_up(E * 4, 128);
    // as many ring slots (up to four) as the shared memory holds
    const int smem_max = device_info().max_smem_optin;
    while (g.nslot > 2 && o + g.nslot * g.slot_bytes > smem_max) --g.nslot;
    // two consumer groups (one token) take alternate slots: an even ring
    if (g.tmax == 1 && (g.nslot & 1)) --g.nslot;
    const int ring = g.nslot * g.slot_bytes;
    g.o_xq += ring; g.o_xd += ring; g.o_bar += ring; g.o_meta += ring; g.o_urec += ring; g.o_gpart += ring;
    g.o_usc += ring; g.o_ent += ring; g.o_selw += ring; g.o_inv += ring; g.o_ys += ring; g.o_misc += ring;
    g.o_base += ring; g.o_part += ring; g.o_bias += ring;
    g.smem_bytes = o + ring;
    return g;
}

// Scratch the selection needs inside its ring slot (T*E doubles x 3 + tables).
static int select_scratch_bytes(int T, int E) { return 3 * T * E * 8 + 4 * 32 * 8 + T * E * 4 + 2 * 128 * 4 + 3 * 256 * 4 + 64 + T * E * 12; }

bool small_path_supported(const moe_config& c, int T) {
    if (T < 1 || T > 4) return false;
    if (c.hidden > 6144 || c.n_experts > 256 || c.n_groups > 32 || c.top_k > 32) return false;
    // bulk copies of whole weight rows start on 16-byte boundaries (int2 rows
    // of a hidden or inter size that is not a multiple of 64 do not)
    if ((c.hidden * c.wbits / 8) % 16 || (c.inter * c.wbits / 8) % 16) return false;
    const SmallGeom g = small_geometry(c, T, device_info().sm_count);
    if (g.rg < 4) return false;  // at least one gate/up row per row group
    if (c.hidden / 32 > kColThreads * kMaxGuBlocks || c.inter / 32 > kColThreads * kMaxDownBlocks) return false;
    if (g.rd < 1 || g.rpc > kMaxOwnedRows || (c.hidden + g.grid - 1) / g.grid > g.rpc) return false;
    if (g.nent > 32 * kMaxEntryWords) return false;
    if (select_scratch_bytes(T, c.n_experts) > g.slot_bytes) return false;
    return g.smem_bytes <= device_info().max_smem_optin;
}

static_assert(kFcDone + 32 * kMaxEntryWords <= (int)(kFusedCtrlBytes / 4), "fused control region");

__global__ void k_fused_ctrl_init(int* ctrl) {
    for (int i = threadIdx.x; i < (int)(kFusedCtrlBytes / 4); i += blockDim.x) ctrl[i] = 0;
    __syncthreads();
    if (threadIdx.x == 0) {
        ctrl[kFcMarker] = (int)(uint32_t)kFcMarkerValue;
        ctrl[kFcMarker + 1] = (int)(uint32_t)(kFcMarkerValue >> 32);
    }
}

cudaError_t launch_fused_ctrl_init(int* ctrl, cudaStream_t s) {
    k_fused_ctrl_init<<<1, 256, 0, s>>>(ctrl);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Router logits (the router row of expert e dotted with x, per token): CTA c
// computes experts c, c + grid, ...; a warp takes eighth w of the hidden
// dimension of one row, each lane holds its weights (float4) in registers
// and keeps four compensated fp32 sums per token (one per float4 component,
// about 2^-48 relative each), folded into fp64; the eighths are added in fp64
// in a fixed order.
// ---------------------------------------------------------------------------
constexpr int kRouterVec = 6;  // float4 of one router row per lane: hidden / 8 / 4 / 32 <= 6

__device__ __forceinline__ void dfacc4_add(DFAcc (&acc)[4], float4 x, float4 w) {
    acc[0].add_prod(x.x, w.x);
    acc[1].add_prod(x.y, w.y);
    acc[2].add_prod(x.z, w.z);
    acc[3].add_prod(x.w, w.w);
}

__device__ __forceinline__ void load_router_row(const float* router_w, int e, int E, int H, int warp, int lane,
                                                float4 (&w)[kRouterVec]) {
    const int n8 = H / 32;  // float4 per eighth
    const float4* wr = reinterpret_cast<const float4*>(router_w + (int64_t)(e < E ? e : 0) * H) + warp * n8;
#pragma unroll
    for (int u = 0; u < kRouterVec; ++u) {
        const int j = lane + 32 * u;
        w[u] = (e < E && j < n8) ? ld_stream_f4(wr + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ---------------------------------------------------------------------------
// Shared-memory layout of the main kernel
// ---------------------------------------------------------------------------
struct SmemPtrs {
    uint8_t* slots;
    uint8_t* xq;  // [tmax][2][nb][16]: each 32-code block in the weights' order, split in halves
    float* xd;    // [tmax][nb]
    uint64_t* full;
    uint64_t* empty;
    uint64_t* routing;  // consumers -> producer: the routing tables are ready
    uint64_t* ufull;    // [2] every consumer warp has written its partials of a unit
    uint64_t* ufree;    // [2] the finisher warp has read them
    uint64_t* gsync;    // the syncing group's warps: their down outputs are in ys
    uint64_t* gexit;    // every consumer warp has left its loop
    uint64_t* rowsin;   // the producer's copy of the CTA's router rows into slot 0 has landed
    uint64_t* ctrl;     // the control snapshot (s.base, misc[8], misc[9]) is in shared memory
    uint64_t* xqin;     // the selecting group has staged every token's Q8_0 codes in xq / xd
    UnitRec* urec;      // [2] the unit to finish
    SlotMeta* meta;
    float* gpart;    // [2][32][2][2][4] gate/up partial dots of a unit: [buffer][pair][gate/up][half][token]
    float* usc;      // [2][32][2] gate/up row scales of a unit
    EntryInfo* ent;  // [nent]
    float* selw;     // [T*k] routing weights
    int* inv;        // [T*k] slot of pair (t, j)
    float* ys;       // [nys][rpc][2] down outputs of the CTA's rows, per column half
    int* misc;       // [0] = routed entries U, [1] routed pairs, [4 + group] units seen,
                     // [8] bit 31 of the router barrier before this call's arrivals,
                     // [9] the control region is initialised
    uint32_t* base;  // [1 + nent] the control counters at the CTA's start: units, done[e]
    double* part;    // [kRouterRound][8][4] router logits per eighth of the hidden dimension
    float* bias;     // [E] router correction bias
};

__device__ __forceinline__ SmemPtrs carve(uint8_t* base, const SmallGeom& g) {
    SmemPtrs s;
    s.slots = base;
    s.xq = base + g.o_xq;
    s.xd = reinterpret_cast<float*>(base + g.o_xd);
    s.full = reinterpret_cast<uint64_t*>(base + g.o_bar);
    s.empty = s.full + kMaxSlots;
    s.routing = s.empty + kMaxSlots;
    s.ufull = s.routing + 1;
    s.ufree = s.ufull + 2;
    s.gsync = s.ufree + 2;
    s.gexit = s.gsync + 1;
    s.rowsin = s.gexit + 1;
    s.ctrl = s.rowsin + 1;
    s.xqin = s.ctrl + 1;
    s.meta = reinterpret_cast<SlotMeta*>(base + g.o_meta);
    s.urec = reinterpret_cast<UnitRec*>(base + g.o_urec);
    s.gpart = reinterpret_cast<float*>(base + g.o_gpart);
    s.usc = reinterpret_cast<float*>(base + g.o_usc);
    s.ent = reinterpret_cast<EntryInfo*>(base + g.o_ent);
    s.selw = reinterpret_cast<float*>(base + g.o_selw);
    s.inv = reinterpret_cast<int*>(base + g.o_inv);
    s.ys = reinterpret_cast<float*>(base + g.o_ys);
    s.misc = reinterpret_cast<int*>(base + g.o_misc);
    s.base = reinterpret_cast<uint32_t*>(base + g.o_base);
    s.part = reinterpret_cast<double*>(base + g.o_part);
    s.bias = reinterpret_cast<float*>(base + g.o_bias);
    return s;
}

// Wait (bounded) until the router barrier has flipped past this call's
// value: every CTA has published its logits.  One thread polls.
__device__ __forceinline__ bool router_barrier_wait(const SmallParams& p, const SmemPtrs& s, uint64_t budget_ns) {
    const uint32_t b0 = (uint32_t)s.misc[8] >> 31;
    const uint64_t t0 = global_timer_ns();
    while (((uint32_t)ld_acquire_gpu(p.ctrl + kFcBarrier) >> 31) == b0) {
        if (global_timer_ns() - t0 > budget_ns) return false;
        __nanosleep(64);
    }
    return true;
}

// Q8_0 of one block of 32 activations held as a float4 by each of 8
// consecutive lanes (the same arithmetic as q8_0_warp): the 4 codes packed
// little-endian into one word, the block scale in d.
__device__ __forceinline__ uint32_t q8_0_octet(float4 v, float& d) {
    float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(kFull, a, o));
    if (!(a >= FLT_MIN)) {
        d = 0.0f;
        return 0u;
    }
    d = __fdiv_rn(a, 127.0f);
    const float id = __fdiv_rn(1.0f, d);
    const float f[4] = {v.x, v.y, v.z, v.w};
    uint32_t w = 0u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float r = roundf(__fmul_rn(f[i], id));
        r = fminf(fmaxf(r, -127.0f), 127.0f);
        w |= ((uint32_t)(int)r & 0xFFu) << (8 * i);
    }
    return w;
}

// Snapshot of the control region that warp 0 takes at the CTA's start: its
// marker and the counters as this CTA finds them (see kFcMarker).  Plain
// loads: what earlier kernels wrote is visible at launch, and this call's
// additions come only after every CTA's router arrival.  Lane l holds the
// counters of entries l, l + 32, ...
struct CtrlSnap {
    uint32_t m0, m1, bar, units;
    uint32_t done[kMaxEntryWords];
};

__device__ __forceinline__ CtrlSnap ctrl_load(const SmallParams& p, int lane, int nent) {
    const volatile int* cv = p.ctrl;
    CtrlSnap c;
    c.m0 = (uint32_t)cv[kFcMarker];
    c.m1 = (uint32_t)cv[kFcMarker + 1];
    c.bar = (uint32_t)cv[kFcBarrier];
    c.units = (uint32_t)cv[kFcUnits];
#pragma unroll
    for (int j = 0; j < kMaxEntryWords; ++j) {
        const int i = lane + 32 * j;
        c.done[j] = i < nent ? (uint32_t)cv[kFcDone + i] : 0u;
    }
    return c;
}

// Warp 0: the snapshot into shared memory (s.base, misc[8], misc[9]); an
// uninitialised region records kErrWorkspace, and the call then only winds
// down (no router arrival, no selection, no publication).
__device__ __forceinline__ void ctrl_store(const SmallParams& p, const SmemPtrs& s, const CtrlSnap& c, int lane,
                                           int nent) {
#pragma unroll
    for (int j = 0; j < kMaxEntryWords; ++j) {
        const int i = lane + 32 * j;
        if (i < nent) s.base[1 + i] = c.done[j];
    }
    if (lane == 0) {
        const bool init = (((uint64_t)c.m1 << 32) | c.m0) == kFcMarkerValue;
        s.base[0] = c.units;
        s.misc[8] = (int)c.bar;
        s.misc[9] = init ? 1 : 0;
        if (blockIdx.x == 0) *p.err = 0;  // before CTA 0's router arrival: no CTA records an error before it
        if (!init) set_error(p.err, kErrWorkspace);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(s.ctrl);
}

// Router rows of CTA c that its producer copies into ring slot 0 (ahead of
// every weight copy) instead of the consumers loading them: the first ones,
// as many as the slot's weight area holds (needs a 16-byte aligned router
// matrix; the flag is set on the host).
__device__ __forceinline__ int router_rows_in_slot(const SmallParams& p, int c, int grid) {
    if (!p.rows_bulk || c >= p.E) return 0;
    const int n_mine = (p.E - 1 - c) / grid + 1;
    const int fit = kSlotWeightBytes / (p.H * 4);
    return min(min(n_mine, fit), kRouterRound);
}

// Every token's Q8_0 codes and scales, as the CTAs published them, into
// shared memory in the weights' order (xq: each block's two 16-byte halves;
// xd): all of a thread's loads are issued before its stores.  The workspace
// was written in this call: L2 loads, after the router barrier's acquire.
template <int WBITS, int TM>
struct XqStage {
    static constexpr int kPer = (TM * 192 + kConsumers - 1) / kConsumers;  // blocks a thread holds at hidden <= 6144
    uint4 lo[kPer], hi[kPer];
    float d[kPer];
    __device__ __forceinline__ void load(const SmallParams& p, int tid) {
        const int nblk = p.T * (p.H / 32);
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int blk = tid + kConsumers * i;
            if (blk < nblk) {
                lo[i] = __ldcg(reinterpret_cast<const uint4*>(p.xq) + 2 * blk);
                hi[i] = __ldcg(reinterpret_cast<const uint4*>(p.xq) + 2 * blk + 1);
                d[i] = __ldcg(p.xd + blk);
            }
        }
    }
    __device__ __forceinline__ void store(const SmallParams& p, const SmemPtrs& s, int tid) {
        const int nb = p.H / 32, nblk = p.T * nb;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int blk = tid + kConsumers * i;
            if (blk < nblk) {
                ActBlock a;
                if constexpr (WBITS == 4) a = act_nibble_order(lo[i], hi[i]);
                else if constexpr (WBITS == 2) a = act_crumb_order(lo[i], hi[i]);
                else a = act_natural(lo[i], hi[i]);
                const int t = blk / nb, b = blk - t * nb;
                *reinterpret_cast<uint4*>(s.xq + ((size_t)(t * 2 + 0) * nb + b) * 16) =
                    make_uint4(a.v[0], a.v[1], a.v[2], a.v[3]);
                *reinterpret_cast<uint4*>(s.xq + ((size_t)(t * 2 + 1) * nb + b) * 16) =
                    make_uint4(a.v[4], a.v[5], a.v[6], a.v[7]);
                s.xd[blk] = d[i];
            }
        }
        // blocks past kPer per thread (hidden above 6144): loaded and stored at once
        for (int blk = tid + kConsumers * kPer; blk < nblk; blk += kConsumers) {
            const uint4 l = __ldcg(reinterpret_cast<const uint4*>(p.xq) + 2 * blk);
            const uint4 h = __ldcg(reinterpret_cast<const uint4*>(p.xq) + 2 * blk + 1);
            ActBlock a;
            if constexpr (WBITS == 4) a = act_nibble_order(l, h);
            else if constexpr (WBITS == 2) a = act_crumb_order(l, h);
            else a = act_natural(l, h);
            const int t = blk / nb, b = blk - t * nb;
            *reinterpret_cast<uint4*>(s.xq + ((size_t)(t * 2 + 0) * nb + b) * 16) =
                make_uint4(a.v[0], a.v[1], a.v[2], a.v[3]);
            *reinterpret_cast<uint4*>(s.xq + ((size_t)(t * 2 + 1) * nb + b) * 16) =
                make_uint4(a.v[4], a.v[5], a.v[6], a.v[7]);
            s.xd[blk] = __ldcg(p.xd + blk);
        }
    }
};

// The consumers' start (all G consumer groups, nthr threads, tid < nthr):
// the Q8_0 of the CTA's share of x's blocks, published to the workspace (xq,
// xd; every CTA stages all of them after the router barrier, XqStage), then
// the CTA's router logits, published to the workspace, from the rows the
// producer copied into `rows` (ring slot 0) and, past those, rows read
// directly.  Ends with the CTA's arrival on the router barrier.  TM bounds
// the tokens: every token's part of x for a router job is loaded together,
// and the tokens' compensated sums advance together.
template <int WBITS, int TM>
__device__ __forceinline__ void consumers_start(const SmallParams& p, const SmemPtrs& s, const uint8_t* rows,
                                                const CtrlSnap& snap, int tid, int nthr) {
    const int warp = tid >> 5, lane = tid & 31, nw = nthr >> 5;
    const int c = blockIdx.x, grid = gridDim.x;
    const int T = p.T, H = p.H, E = p.E, nb = H / 32;
    const int n_mine = c < E ? (E - 1 - c) / grid + 1 : 0;  // router rows of this CTA
    const int n_slot = router_rows_in_slot(p, c, grid);     // of which the producer copies these
    const float bias_v = tid < E ? __ldg(p.bias + tid) : 0.f;  // stored below: its load overlaps x's
    // Q8_0 of x: the CTAs share the blocks (CTA c takes the steps of 4
    // blocks [c S / grid, (c + 1) S / grid)) and publish the codes and scales
    // to the workspace (xq, xd); after the router barrier every CTA stages
    // all of them in shared memory (XqStage).  A warp takes 4 blocks at a
    // time (8 lanes, a float4 each).
    {
        const int nblk = T * nb, nstep = (nblk + 3) / 4, l8 = lane & 7;
        const int st0 = (int)((int64_t)c * nstep / grid), st1 = (int)((int64_t)(c + 1) * nstep / grid);
        for (int st = st0 + warp; st < st1; st += nw) {
            const int blk = 4 * st + (lane >> 3);
            const float4 v = blk < nblk ? __ldg(reinterpret_cast<const float4*>(p.x) + (int64_t)blk * 8 + l8)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
            float d;
            const uint32_t q = q8_0_octet(v, d);  // natural codes 4 l8 .. 4 l8 + 3
            if (blk < nblk) {
                reinterpret_cast<uint32_t*>(p.xq)[(int64_t)blk * 8 + l8] = q;
                if (l8 == 0) p.xd[blk] = d;
            }
        }
    }
    if (tid < E) s.bias[tid] = bias_v;  // read by the selection
    for (int e = tid + nthr; e < E; e += nthr) s.bias[e] = __ldg(p.bias + e);
    if (warp == 0) ctrl_store(p, s, snap, lane, p.g.nent);
    // router logits, kRouterRound rows at a time: job = (row of the round,
    // eighth of the hidden dimension)
    const int n8 = H / 32;
    bool rows_waited = n_slot == 0;
    for (int r0 = 0; r0 < n_mine; r0 += kRouterRound) {
        const int nr = min(kRouterRound, n_mine - r0);
        for (int job = warp; job < nr * 8; job += nw) {
            const int i = job >> 3, w8 = job & 7, e = c + grid * (r0 + i);
            float4 w[kRouterVec];
            if (r0 + i < n_slot) {
                if (!rows_waited) {
                    int ok = 1;
                    if (lane == 0) ok = mbar_wait_ns(s.rowsin, 0, kSlackWaits * p.wait_ns) ? 1 : 0;
                    if (!__shfl_sync(kFull, ok, 0) && lane == 0) set_error(p.err, kErrTimeout);
                    rows_waited = true;
                }
                const float4* wr = reinterpret_cast<const float4*>(rows + (size_t)(r0 + i) * H * 4) + w8 * n8;
#pragma unroll
                for (int u = 0; u < kRouterVec; ++u) {
                    const int j = lane + 32 * u;
                    w[u] = j < n8 ? wr[j] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            } else {
                load_router_row(p.router_w, e, E, H, w8, lane, w);
            }
            float4 xv[TM][kRouterVec];
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                const float4* xr = reinterpret_cast<const float4*>(p.x + (int64_t)(t < T ? t : 0) * H) + w8 * n8;
#pragma unroll
                for (int u = 0; u < kRouterVec; ++u) {
                    const int j = lane + 32 * u;
                    xv[t][u] = (t < T && j < n8) ? __ldg(xr + j) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            // every token's four compensated sums advance together (4 TM
            // independent chains; each sum sees its terms in the same order)
            DFAcc acc[TM][4];
#pragma unroll
            for (int u = 0; u < kRouterVec; ++u)
#pragma unroll
                for (int t = 0; t < TM; ++t) dfacc4_add(acc[t], xv[t][u], w[u]);
#pragma unroll
            for (int t = 0; t < TM; ++t) {
                if (t >= T) break;  // the same for the whole warp
                double v = (acc[t][0].value() + acc[t][1].value()) + (acc[t][2].value() + acc[t][3].value());
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
                if (lane == 0) s.part[(i * 8 + w8) * 4 + t] = v;
            }
        }
        named_barrier(3, nthr);
        if (tid < nr * T) {
            const int i = tid / T, t = tid - i * T;
            double v = 0.0;
#pragma unroll
            for (int k = 0; k < 8; ++k) v += s.part[(i * 8 + k) * 4 + t];
            // the sigmoid here, off the selection's path
            p.logits[(int64_t)t * E + c + grid * (r0 + i)] = 1.0 / (1.0 + exp(-v));
        }
        named_barrier(3, nthr);
    }
    // every consumer thread's logits are written: the CTA's arrival (CTA 0
    // adds 2^31 - (grid - 1), the others 1: bit 31 flips at the last one)
    named_barrier(3, nthr);
    if (tid == 0 && s.misc[9]) {
        const int add = c == 0 ? (int)(0x80000000u - (uint32_t)(grid - 1)) : 1;
        red_add_release_gpu(p.ctrl + kFcBarrier, add);
    }
}

// ---------------------------------------------------------------------------
// Producer: the whole warp runs the schedule in lockstep; lane 0 owns the
// barriers, lanes 0..3 issue one copy each, all lanes help poll.
// ---------------------------------------------------------------------------
struct Copy {
    const void* src;
    uint32_t bytes;
    uint32_t dst;  // byte offset in the slot
    bool stream;   // read-once weights: L2 evict-first
    int first;     // windows: slot offset of the first requested value
};

__device__ __forceinline__ Copy no_copy() { return Copy{nullptr, 0u, 0u, false, 0}; }

// A 16-byte aligned window over `count` fp32 values at src, placed at slot
// offset dst.
__device__ __forceinline__ Copy window(const float* src, int count, uint32_t dst) {
    const uintptr_t lo = reinterpret_cast<uintptr_t>(src);
    const uintptr_t hi = lo + (uintptr_t)count * 4u;
    const uintptr_t alo = lo & ~uintptr_t(15), ahi = (hi + 15) & ~uintptr_t(15);
    return Copy{reinterpret_cast<const void*>(alo), count > 0 ? (uint32_t)(ahi - alo) : 0u, dst, false,
                (int)dst + (int)(lo - alo)};
}

struct Producer {
    const SmallParams& p;
    const SmemPtrs& s;
    const int lane;
    const int groups;  // consumer groups (each takes every groups-th ring slot)
    uint64_t pol;
    int slot = 0;
    int units = 0;     // gate/up units issued (their ordinals stamp the items)
    uint32_t pe = 1;  // parity to wait on the empty barriers (fresh ring: all empty)
    bool aborted = false;
    bool need_proxy_fence = false;  // set after acquiring data that later copies read
    uint32_t issued_mask = 0, issued_par = 0;
    uint32_t rdy0 = 0, rdy1 = 0, rdy2 = 0, rdy3 = 0, rdy4 = 0;  // entries whose h codes are all published

    __forceinline__ __device__ Producer(const SmallParams& p_, const SmemPtrs& s_, int lane_, int groups_)
        : p(p_), s(s_), lane(lane_), groups(groups_) {
        pol = l2_evict_first_policy();
    }

    __forceinline__ __device__ void fail() {
        if (lane == 0) set_error(p.err, kErrTimeout);
        aborted = true;
    }

    __forceinline__ __device__ SlotMeta blank(int kind) const {
        SlotMeta m;
        m.kind = kind;
        m.entry = 0;
        m.expert = -1;
        m.row0 = 0;
        m.nrows = 0;
        m.n = 0;
        m.slot0 = 0;
        m.blk = 0;
        m.last = 0;
        m.off_a = 0;
        m.off_b = 0;
        m.uc = 0;
        for (int i = 0; i < 4; ++i) m.tok[i] = 0;
        return m;
    }

    __forceinline__ __device__ void set_entry(SlotMeta& m, int entry, const EntryInfo& ei) const {
        m.entry = entry;
        m.expert = ei.expert;
        m.n = ei.n;
        m.slot0 = ei.slot0;
        for (int i = 0; i < 4; ++i) m.tok[i] = ei.tok[i];
    }

    // Hand one item over: wait for its slot, publish the meta, arm the full
    // barrier with the byte count and start the copies (lane i issues copy i).
    __forceinline__ __device__ bool push(const SlotMeta& m, const Copy& c0, const Copy& c1, const Copy& c2,
                                         const Copy& c3) {
        if (aborted) return false;
        int ok = 1;
        if (lane == 0) ok = mbar_wait_ns(&s.empty[slot], pe, p.wait_ns) ? 1 : 0;
        ok = __shfl_sync(kFull, ok, 0);
        __syncwarp();
        if (!ok) {
            fail();
            return false;
        }
        uint8_t* dst = s.slots + (size_t)slot * p.g.slot_bytes;
        if (lane == 0) {
            s.meta[slot] = m;
            const uint32_t total = c0.bytes + c1.bytes + c2.bytes + c3.bytes;
            if (total == 0) mbar_arrive(&s.full[slot]);
            else mbar_arrive_expect_tx(&s.full[slot], total);
        }
        __syncwarp();
        if (lane < 4) {
            const void* src = lane == 0 ? c0.src : lane == 1 ? c1.src : lane == 2 ? c2.src : c3.src;
            const uint32_t bytes = lane == 0 ? c0.bytes : lane == 1 ? c1.bytes : lane == 2 ? c2.bytes : c3.bytes;
            const uint32_t off = lane == 0 ? c0.dst : lane == 1 ? c1.dst : lane == 2 ? c2.dst : c3.dst;
            const bool stream = lane == 0 ? c0.stream : lane == 1 ? c1.stream : lane == 2 ? c2.stream : c3.stream;
            if (bytes) {
                if (need_proxy_fence) fence_proxy_async_global();
                if (stream) bulk_g2s(dst + off, src, bytes, &s.full[slot], pol);
                else bulk_g2s_nohint(dst + off, src, bytes, &s.full[slot]);
            }
        }
        __syncwarp();
        need_proxy_fence = false;
        issued_mask |= 1u << slot;
        issued_par = (issued_par & ~(1u << slot)) | ((pe ^ 1u) << slot);
        if (++slot == p.g.nslot) {
            slot = 0;
            pe ^= 1u;
        }
        return true;
    }

    __forceinline__ __device__ bool marker(int kind) {
        return push(blank(kind), no_copy(), no_copy(), no_copy(), no_copy());
    }

    // Chunk ch of gate/up unit blk of an entry: rg rows of Wg and of Wu and
    // their row scales.
    __forceinline__ __device__ bool gateup(int entry, const EntryInfo& ei, int blk, int ch) {
        const SmallGeom& g = p.g;
        SlotMeta m = blank(kItemGateUp);
        set_entry(m, entry, ei);
        m.blk = blk;
        m.last = ch == g.cpu - 1;
        m.row0 = blk * kUnit + ch * g.rg;
        m.nrows = g.rg;
        const moe_experts& ex = entry ? p.routed : p.shared;
        const int64_t r = (int64_t)(entry ? ei.expert : 0) * p.I + m.row0;
        const int64_t rowH = (int64_t)p.H * p.wbits / 8;
        const uint32_t wb = (uint32_t)(g.rg * rowH);
        const Copy c0{ex.w_gate + r * rowH, wb, 0u, true, 0};
        const Copy c1{ex.w_up + r * rowH, wb, wb, true, 0};
        const Copy c2 = window(ex.s_gate + r, g.rg, kSlotWeightBytes);
        const Copy c3 = window(ex.s_up + r, g.rg, kSlotWeightBytes + kScaleWin);
        m.off_a = c2.first;
        m.off_b = c3.first;
        m.uc = units;
        if (m.last) ++units;
        return push(m, c0, c1, c2, c3);
    }

    // nrows down rows of an entry starting at row0, with the entry's h codes
    // and scales and the rows' scales.  lrow = row0 - first owned row.
    __forceinline__ __device__ bool down(int entry, const EntryInfo& ei, int row0, int nrows, int lrow) {
        const SmallGeom& g = p.g;
        SlotMeta m = blank(kItemDown);
        set_entry(m, entry, ei);
        m.row0 = row0;
        m.nrows = nrows;
        m.blk = lrow;
        const moe_experts& ex = entry ? p.routed : p.shared;
        const int64_t eo = entry ? ei.expert : 0;
        const int64_t rowI = (int64_t)p.I * p.wbits / 8;
        const int nbI = p.I / 32;
        const Copy c0{ex.w_down + (eo * p.H + row0) * rowI, (uint32_t)(nrows * rowI), 0u, true, 0};
        const Copy c1{p.hq + (int64_t)ei.slot0 * p.I, (uint32_t)(ei.n * p.I), (uint32_t)kSlotWeightBytes, false, 0};
        const Copy c2 = window(p.hd + (int64_t)ei.slot0 * nbI, ei.n * nbI, kSlotWeightBytes + g.a_hd);
        const Copy c3 = window(ex.s_down + eo * p.H + row0, nrows, kSlotWeightBytes + g.a_sd);
        m.off_a = c2.first;
        m.off_b = c3.first;
        return push(m, c0, c1, c2, c3);
    }

    // Wait until every unit of entry e has published its h codes.  Each poll
    // reads all entries' counters at once (one round trip for the warp).
    __forceinline__ __device__ bool is_ready(int e) const {
        const int wi = e >> 5;
        const uint32_t w = wi == 0 ? rdy0 : wi == 1 ? rdy1 : wi == 2 ? rdy2 : wi == 3 ? rdy3 : rdy4;
        return (w >> (e & 31)) & 1u;
    }

    __forceinline__ __device__ bool entry_done(int i, int U) const {
        return i <= U && (uint32_t)ld_acquire_gpu(p.ctrl + kFcDone + i) - s.base[1 + i] >= (uint32_t)(p.g.nu * s.ent[i].n);
    }

    // One poll of every entry's counter (one round trip for the warp): the
    // entries found complete need no wait later.
    __forceinline__ __device__ void poll_entries(int U) {
        const bool f0 = entry_done(lane, U), f1 = entry_done(lane + 32, U), f2 = entry_done(lane + 64, U);
        const bool f3 = entry_done(lane + 96, U), f4 = entry_done(lane + 128, U);
        rdy0 |= __ballot_sync(kFull, f0);
        rdy1 |= __ballot_sync(kFull, f1);
        rdy2 |= __ballot_sync(kFull, f2);
        rdy3 |= __ballot_sync(kFull, f3);
        rdy4 |= __ballot_sync(kFull, f4);
        need_proxy_fence = true;
        __syncwarp();  // the polling lanes' acquires order the copying lanes' reads
    }

    // Wait until every unit of entry e has published its h codes.  Each poll
    // reads all entries' counters at once (one round trip for the warp).
    __forceinline__ __device__ bool wait_entry(int e, int U) {
        if (is_ready(e)) return true;
        need_proxy_fence = true;
        const uint64_t t0 = global_timer_ns();
        while (global_timer_ns() - t0 <= p.wait_ns) {
            const bool f0 = entry_done(lane, U), f1 = entry_done(lane + 32, U), f2 = entry_done(lane + 64, U);
            const bool f3 = entry_done(lane + 96, U), f4 = entry_done(lane + 128, U);
            rdy0 = __ballot_sync(kFull, f0);
            rdy1 = __ballot_sync(kFull, f1);
            rdy2 = __ballot_sync(kFull, f2);
            rdy3 = __ballot_sync(kFull, f3);
            rdy4 = __ballot_sync(kFull, f4);
            if (is_ready(e)) {
                __syncwarp();  // the polling lanes' acquires order the copying lanes' reads
                return true;
            }
            __nanosleep(128);
        }
        fail();
        return false;
    }

    // One DONE marker per consumer group (consecutive slots belong to
    // different groups), carrying the CTA's unit count.  After a timeout this
    // runs with `aborted` set: each marker is handed over if a slot frees up in
    // time (otherwise that group times out on its own).
    __forceinline__ __device__ void finish() {
        for (int gi = 0; gi < groups; ++gi) {
            int ok = 0;
            if (lane == 0 && mbar_wait_ns(&s.empty[slot], pe, p.wait_ns)) {
                s.meta[slot].kind = kItemDone;
                s.meta[slot].uc = units;
                mbar_arrive(&s.full[slot]);
                ok = 1;
            }
            ok = __shfl_sync(kFull, ok, 0);
            if (!ok) {
                if (lane == 0) set_error(p.err, kErrTimeout);
                return;
            }
            issued_mask |= 1u << slot;
            issued_par = (issued_par & ~(1u << slot)) | ((pe ^ 1u) << slot);
            if (++slot == p.g.nslot) {
                slot = 0;
                pe ^= 1u;
            }
        }
    }

    // Before the CTA exits: wait (bounded) for every copy it issued.
    __forceinline__ __device__ void drain() {
        if (lane != 0) return;
        for (int i = 0; i < p.g.nslot; ++i)
            if ((issued_mask >> i) & 1u) mbar_wait_ns(&s.full[i], (issued_par >> i) & 1u, p.wait_ns);
    }
};

// ---------------------------------------------------------------------------
// Consumer items
// ---------------------------------------------------------------------------
// Barrier of one consumer group's warps (group 0 runs the selection).
__device__ __forceinline__ void group_sync(int group) { named_barrier(1 + group, kConsumers); }
__device__ __forceinline__ void consumers_sync() { group_sync(0); }

// (ka, ia) ranks before (kb, ib): larger key, ties to the lower index.
// Branch-free, so that unrolled compare loops pipeline their loads.
__device__ __forceinline__ bool beats(unsigned long long ka, int ia, unsigned long long kb, int ib) {
    return (ka > kb) | ((ka == kb) & (ia < ib));
}

// Arg-max of 64-bit keys over the warp, ties to the lower index: the key's
// halves go through the warp max-reduction one after the other, the index
// through a min-reduction over the lanes that hold the maximum.
__device__ __forceinline__ int warp_argmax_u64(unsigned long long key, int idx) {
    const uint32_t hi = (uint32_t)(key >> 32), lo = (uint32_t)key;
    const uint32_t mh = __reduce_max_sync(kFull, hi);
    const uint32_t ml = __reduce_max_sync(kFull, hi == mh ? lo : 0u);
    return (int)__reduce_min_sync(kFull, (hi == mh && lo == ml) ? (uint32_t)idx : 0x7FFFFFFFu);
}

// Bitonic sort of the warp's 32 (key, index) pairs, best first (larger key,
// ties to the lower index): lane r ends with the r-th best.
__device__ __forceinline__ void warp_sort_desc(unsigned long long& k, int& i, int lane) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int st = size >> 1; st > 0; st >>= 1) {
            const unsigned long long ok = __shfl_xor_sync(kFull, k, st);
            const int oi = __shfl_xor_sync(kFull, i, st);
            const bool keep_best = ((lane & st) == 0) == ((lane & size) == 0);
            const bool other_better = beats(ok, oi, k, i);
            if (keep_best == other_better) {
                k = ok;
                i = oi;
            }
        }
    }
}

// SELECT: wait for every router item, then route all tokens and bucket them
// into this CTA's tables (the same in every CTA; CTA 0 also publishes them to
// the workspace).  Same decisions as the multi-kernel router and the
// reference: group score = sum of the two largest c = s + bias, keep
// topk_groups groups, then top_k experts in descending c, ties to the lower
// index, w = s / sum(s) * rsf with the unbiased s.  Keys are order-preserving
// 64-bit images of c.  Every decision is a rank computed by one thread with
// independent compares, in short phases that keep all warps busy:
//   1. s, c, keys;  2. each expert's rank inside its group (the best
//   kc = min(max(top_k, 2), group size) of each group are listed in order);
//   3. group keys, then each group's rank (kept = rank < topk_groups);
//   4. each listed expert of a kept group: its rank among the listed experts
//   of the kept groups (only those can reach the top_k);  5. bucketing.
// With groups of 32 experts (one warp each) phases 2-4 use warp arg-max
// rounds instead: k rounds list each group's best k in order, and one warp
// per token ranks the kept groups' lists with shuffles.
// The producer is released as soon as the tables it needs are written; the
// routing weights, needed only by the combine, come last.  The item's ring
// slot is the scratch.
__device__ __forceinline__ void do_select(const SmallParams& p, const SmemPtrs& s, uint8_t* scratch, int tid) {
    const int E = p.E, T = p.T, k = p.k, G = p.G, per = E / G, tg = p.tg;
    const int TE = T * E;
    const int kc = min(max(k, 2), per);  // listed experts per group
    const int kk = min(k, per);          // of which can reach the top_k
    const bool publish = blockIdx.x == 0;
    const bool fast = per == 32 && G <= kConsumerWarps && tg <= kMaxKeptFast && tg * kk <= 32;
    double* sc = reinterpret_cast<double*>(scratch);                         // [T][E] c = s + bias
    double* ss = sc + TE;                                                     // [T][E] s
    unsigned long long* key = reinterpret_cast<unsigned long long*>(ss + TE);  // [T][E] order key of c
    unsigned long long* gkey = key + TE;                                      // [T][32] group-score keys
    int* cand = reinterpret_cast<int*>(gkey + 4 * 32);                        // [T][G][kc] listed experts
    int* kg = cand + TE;                                                      // [T][32] kept groups
    int* sel = kg + 4 * 32;                                                   // [T][32] picks, by rank
    int* cnt = sel + 4 * 32;                                                  // [E]
    int* off = cnt + 256;                                                     // [E] exclusive scan of counts
    int* ent = off + 256;                                                     // [E] entry index
    int* wsum = ent + 256;                                                    // [8][2] warp totals
    unsigned long long* lkey = reinterpret_cast<unsigned long long*>(wsum + 16);  // [T][tg*kk] listed keys
    int* lid = reinterpret_cast<int*>(lkey + T * p.tg * min(k, per));            // [T][tg*kk] listed ids
    const int warp = tid >> 5, lane = tid & 31;
    // the logits are every CTA's: the router barrier has completed
    // 1. s, c and keys
#pragma unroll 1
    for (int i = tid; i < TE; i += kConsumers) {
        const double sv = __ldcg(p.logits + i);  // s = sigmoid(logit), published by the row's CTA
        const double cv = sv + (double)s.bias[i % E];
        ss[i] = sv;
        sc[i] = cv;
        key[i] = order_key(cv);
    }
#pragma unroll 1
    for (int e = tid; e < E; e += kConsumers) cnt[e] = 0;
    consumers_sync();
    if (fast) {
        // GLM-like shape: warp g owns group g (32 experts, one per lane).
        // 2. each (token, group): its best two experts by two warp arg-max
        // rounds (larger key, ties to the lower index) give the group score
        if (warp < G) {
            const int g = warp, e = g * 32 + lane;
#pragma unroll 1
            for (int t = 0; t < T; ++t) {
                const unsigned long long kv = key[(size_t)t * E + e];
                const int b1 = warp_argmax_u64(kv, e);
                const int b2 = warp_argmax_u64(e == b1 ? 0ull : kv, e == b1 ? 0x7FFFFFFF : e);
                if (lane == 0) gkey[t * 32 + g] = order_key(sc[(size_t)t * E + b1] + sc[(size_t)t * E + b2]);
            }
        }
        consumers_sync();
        // 3.-4. one warp per token: each group's rank among the token's groups
        // (kept = rank < topk_groups), then k arg-max rounds over the kept
        // groups' experts (lane l holds expert l of each kept group); the
        // picks come out best first
        if (warp < T) {
            const int t = warp;
            const unsigned long long gk = lane < G ? gkey[t * 32 + lane] : 0ull;
            int grank = 0;
#pragma unroll 1
            for (int g2 = 0; g2 < G; ++g2) grank += beats(gkey[t * 32 + g2], g2, gk, lane) ? 1 : 0;
            uint32_t kept = __ballot_sync(kFull, lane < G && grank < tg);
            unsigned long long ck[kMaxKeptFast];
            int ce[kMaxKeptFast];
#pragma unroll
            for (int q = 0; q < kMaxKeptFast; ++q) {  // kept groups in index order (the order does not change the picks)
                const int g = kept ? __ffs(kept) - 1 : -1;
                kept &= kept - 1;
                ce[q] = g >= 0 ? g * 32 + lane : 0x7FFFFFFF;
                ck[q] = g >= 0 ? key[(size_t)t * E + ce[q]] : 0ull;
            }
#pragma unroll 1
            for (int j = 0; j < k; ++j) {
                unsigned long long bk = ck[0];
                int be = ce[0];
#pragma unroll
                for (int q = 1; q < kMaxKeptFast; ++q)
                    if (beats(ck[q], ce[q], bk, be)) {
                        bk = ck[q];
                        be = ce[q];
                    }
                const int win = warp_argmax_u64(bk, be);
#pragma unroll
                for (int q = 0; q < kMaxKeptFast; ++q)
                    if (ce[q] == win) {  // taken: out of the later rounds
                        ck[q] = 0ull;
                        ce[q] = 0x7FFFFFFF;
                    }
                if (lane == 0) sel[t * 32 + j] = win;
            }
        }
        consumers_sync();
    } else {
        // 2. rank inside the group
    #pragma unroll 1
        for (int i = tid; i < TE; i += kConsumers) {
            const int t = i / E, e = i - t * E, g = e / per;
            const unsigned long long* kt = key + (size_t)t * E + g * per;
            const unsigned long long ke = kt[e - g * per];
            int rank = 0;
    #pragma unroll 1
            for (int r2 = 0; r2 < per; ++r2) rank += beats(kt[r2], g * per + r2, ke, e) ? 1 : 0;
            if (rank < kc) cand[(t * G + g) * kc + rank] = e;
        }
        consumers_sync();
        // 3. group keys, then group ranks
        if (tid < T * G) {
            const int t = tid / G, g = tid - t * G;
            const int* cg = cand + (t * G + g) * kc;
            gkey[t * 32 + g] = order_key(sc[(size_t)t * E + cg[0]] + sc[(size_t)t * E + cg[1]]);
        }
        consumers_sync();
        if (tid < T * G) {
            const int t = tid / G, g = tid - t * G;
            const unsigned long long kgk = gkey[t * 32 + g];
            int rank = 0;
    #pragma unroll 1
            for (int g2 = 0; g2 < G; ++g2) rank += beats(gkey[t * 32 + g2], g2, kgk, g) ? 1 : 0;
            if (rank < tg) kg[t * 32 + rank] = g;
        }
        consumers_sync();
        // 4. final ranks among the listed experts of the kept groups (their keys
        // and ids gathered first into one contiguous list per token)
        const int nl = tg * kk;
    #pragma unroll 1
        for (int i = tid; i < T * nl; i += kConsumers) {
            const int t = i / nl, rem = i - t * nl, q = rem / kk, r = rem - q * kk;
            const int e = cand[(t * G + kg[t * 32 + q]) * kc + r];
            lkey[i] = key[(size_t)t * E + e];
            lid[i] = e;
        }
        consumers_sync();
    #pragma unroll 1
        for (int i = tid; i < T * nl; i += kConsumers) {
            const int t = i / nl;
            const unsigned long long* lk = lkey + t * nl;
            const int* li = lid + t * nl;
            const unsigned long long ke = lkey[i];
            const int e = lid[i];
            int rank = 0;
    #pragma unroll 1
            for (int j = 0; j < nl; ++j) rank += beats(lk[j], li[j], ke, e) ? 1 : 0;
            if (rank < k) sel[t * 32 + rank] = e;
        }
        consumers_sync();
    }
    // 4b. adaptive expert top-p (one warp per token): the dropped picks leave
    // sel as -1 before the bucketing, and the weights are final here
    const bool topp_on = p.topp > 0.f && p.topp < 1.f;
    if (topp_on) {
        if (warp < T) {
            const int t = warp;
            const int e = lane < k ? sel[t * 32 + lane] : 0;
            const double sj = lane < k ? ss[(size_t)t * E + e] : 0.0;
            double ssum = 0.0;
            for (int j = 0; j < k; ++j) ssum += __shfl_sync(kFull, sj, j);  // pick order
            double skept;
            const bool keep = topp_keep(sj, ssum, k, p.topp, lane, &skept);
            if (lane < k) {
                const float wv = keep ? (float)(sj / skept * (double)p.rsf) : 0.f;
                s.selw[t * k + lane] = wv;
                if (!keep) sel[t * 32 + lane] = -1;
                if (publish) {
                    p.idx[(int64_t)t * k + lane] = keep ? e : -1;
                    p.w[(int64_t)t * k + lane] = wv;
                }
            }
        }
        consumers_sync();
    }
    // 4c. expert parallelism: the picks outside [ep_lo, ep_hi) are computed by
    // another call; the routing and the weights are published as they are,
    // then those picks leave sel as -1 (in no bucket, skipped by the combine)
    const bool ep_on = p.ep_lo > 0 || p.ep_hi < E;
    if (ep_on) {
        if (!topp_on && warp < T && lane < k) {
            const int t = warp;
            double ssum = 0.0;
            for (int j = 0; j < k; ++j) ssum += ss[(size_t)t * E + sel[t * 32 + j]];
            const int e = sel[t * 32 + lane];
            const float wv = (float)(ss[(size_t)t * E + e] / ssum * (double)p.rsf);
            s.selw[t * k + lane] = wv;
            if (publish) {
                p.idx[(int64_t)t * k + lane] = e;
                p.w[(int64_t)t * k + lane] = wv;
            }
        }
        consumers_sync();
        if (warp < T && lane < k) {
            const int e = sel[warp * 32 + lane];
            if (e >= 0 && (e < p.ep_lo || e >= p.ep_hi)) sel[warp * 32 + lane] = -1;
        }
        consumers_sync();
    }
    // 5. bucketing (a dropped pick, sel -1, is in no bucket: inv -1)
    const int n = T * k;
    if (n <= 32) {
        // one warp, lane = pick t * k + j: same-expert lanes found with a
        // match, positions from counts over the other lanes
        if (warp == 0) {
            const int e_in = lane < n ? sel[(lane / k) * 32 + lane % k] : -1;
            const bool act = e_in >= 0;
            const int e = act ? e_in : 0x7FFFFFFF;
            // one token: the picks are distinct experts
            const uint32_t same = T == 1 ? (1u << lane) : __match_any_sync(kFull, e);
            const int lead = __ffs(same) - 1;
            const int rank = __popc(same & ((1u << lane) - 1u));  // earlier picks (tokens) of this expert
            int less = 0, dless = 0;  // picks / distinct experts below e
#pragma unroll 8
            for (int l2 = 0; l2 < n; ++l2) {  // partly unrolled: the shuffles pipeline (lanes >= n hold no pick)
                const int e2 = __shfl_sync(kFull, e, l2);
                const int lead2 = __shfl_sync(kFull, lead, l2);
                less += e2 < e ? 1 : 0;
                dless += (e2 < e && lead2 == l2) ? 1 : 0;
            }
            if (act) {
                const int pos = less + rank;
                s.inv[lane] = pos;
                if (lane == lead) {
                    EntryInfo& ei = s.ent[1 + dless];
                    ei.expert = e;
                    ei.slot0 = less;
                    ei.n = __popc(same);
                }
                if (publish) {
                    p.perm[pos] = lane;
                    p.inv_perm[lane] = pos;
                    if (lane == lead) p.active[1 + dless] = e;
                }
            } else if (lane < n) {  // dropped by the top-p
                s.inv[lane] = -1;
                if (publish) p.inv_perm[lane] = -1;
            }
            const int n_act = __popc(__ballot_sync(kFull, act));  // routed pairs
            if (publish && lane >= n_act && lane < n) p.perm[lane] = -1;
            if (lane == 0) s.misc[1] = n_act;
            __syncwarp();
            if (act && rank < 4) s.ent[1 + dless].tok[rank] = lane / k;
            const int U = __popc(__ballot_sync(kFull, act && lane == lead));
            if (lane == 0) {
                s.misc[0] = U;
                if (publish) p.active[0] = U;
                EntryInfo& e0 = s.ent[0];
                e0.expert = -1;
                e0.slot0 = n;
                e0.n = T;
#pragma unroll 1
                for (int i = 0; i < 4; ++i) e0.tok[i] = i < T ? i : 0;
            }
        }
        consumers_sync();  // every table the producer reads is written
        if (tid == 0) mbar_arrive(s.routing);
        if (publish) {
            // counts and offsets of every expert: the first entry (entries are
            // in ascending expert order) whose expert is not below e
            const int U = s.misc[0], n_act = s.misc[1];
#pragma unroll 1
            for (int e = tid; e <= E; e += kConsumers) {
                int lo = 1, hi = U + 1;
#pragma unroll 1
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (s.ent[mid].expert < e) lo = mid + 1;
                    else hi = mid;
                }
                const bool in = lo <= U;
                p.offsets[e] = in ? s.ent[lo].slot0 : n_act;
                if (e < E) p.counts[e] = (in && s.ent[lo].expert == e) ? s.ent[lo].n : 0;
            }
        }
    } else {
        if (tid < n && sel[(tid / k) * 32 + tid % k] >= 0) atomicAdd(&cnt[sel[(tid / k) * 32 + tid % k]], 1);
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
#pragma unroll 1
            for (int w = 0; w < warp; ++w) {
                b1 += wsum[w * 2];
                b2 += wsum[w * 2 + 1];
            }
            if (tid < E) {
                const int o = b1 + a1 - cv, ai = b2 + a2 - nz;
                off[tid] = o;
                ent[tid] = ai;
                if (cv > 0) {
                    EntryInfo& ei = s.ent[1 + ai];
                    ei.expert = tid;
                    ei.slot0 = o;
                    ei.n = cv;
                }
                if (tid == E - 1) {
                    s.misc[0] = ai + nz;
                    s.misc[1] = o + cv;  // routed pairs
                }
                if (publish) {
                    p.offsets[tid] = o;
                    p.counts[tid] = cv;
                    if (cv > 0) p.active[1 + ai] = tid;
                    if (tid == E - 1) {
                        p.offsets[E] = o + cv;
                        p.active[0] = ai + nz;
                    }
                }
            }
            if (tid == 0) {
                EntryInfo& e0 = s.ent[0];
                e0.expert = -1;
                e0.slot0 = n;
                e0.n = T;
#pragma unroll 1
                for (int i = 0; i < 4; ++i) e0.tok[i] = i < T ? i : 0;
            }
        }
        consumers_sync();
        if (publish && tid < n && tid >= s.misc[1]) p.perm[tid] = -1;  // the dropped pairs' tail
        if (tid < n && sel[(tid / k) * 32 + tid % k] < 0) {  // dropped by the top-p
            s.inv[tid] = -1;
            if (publish) p.inv_perm[tid] = -1;
        } else if (tid < n) {
            const int t = tid / k;
            const int e = sel[t * 32 + tid % k];
            int rank = 0;
#pragma unroll 1
            for (int t2 = 0; t2 < t; ++t2)
#pragma unroll 1
                for (int j2 = 0; j2 < k; ++j2) rank += sel[t2 * 32 + j2] == e ? 1 : 0;
            const int pos = off[e] + rank;
            s.inv[tid] = pos;
            if (rank < 4) s.ent[1 + ent[e]].tok[rank] = t;
            if (publish) {
                p.perm[pos] = tid;
                p.inv_perm[tid] = pos;
            }
        }
        consumers_sync();  // every table the producer reads is written
        if (tid == 0) mbar_arrive(s.routing);
    }
    // routing weights from the unbiased sigmoid, summed in pick order (with the
    // top-p they were written before the bucketing)
    if (!topp_on && !ep_on && warp < T && lane < k) {
        const int t = warp;
        double ssum = 0.0;
#pragma unroll 8
        for (int j = 0; j < k; ++j) ssum += ss[(size_t)t * E + sel[t * 32 + j]];
        const int e = sel[t * 32 + lane];
        const float wv = (float)(ss[(size_t)t * E + e] / ssum * (double)p.rsf);
        s.selw[t * k + lane] = wv;
        if (publish) {
            p.idx[(int64_t)t * k + lane] = e;
            p.w[(int64_t)t * k + lane] = wv;
        }
    }
}

// m.tok[i] with a run-time i, without indexing a local array.
__device__ __forceinline__ int tok_at(const SlotMeta& m, int i) {
    return i == 0 ? m.tok[0] : i == 1 ? m.tok[1] : i == 2 ? m.tok[2] : m.tok[3];
}

template <int WBITS>
__device__ __forceinline__ WBlock<WBITS> load_block_smem(const uint8_t* row, int b) {
    WBlock<WBITS> w;
    if constexpr (WBITS == 4) {
        w.a = *reinterpret_cast<const uint4*>(row + 16 * b);
        w.b = make_uint4(0, 0, 0, 0);
    } else if constexpr (WBITS == 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(row + 8 * b);
        w.a = make_uint4(v.x, v.y, 0, 0);
        w.b = make_uint4(0, 0, 0, 0);
    } else {
        w.a = *reinterpret_cast<const uint4*>(row + 32 * b);
        w.b = *reinterpret_cast<const uint4*>(row + 32 * b + 16);
    }
    return w;
}

// ---- gate/up chunk: rg row pairs of one unit -> partial dots; the unit's
// last chunk turns the 32 rows into h = silu(g) * u, quantises the block and
// publishes it ----
template <int WBITS, int TM>
__device__ __forceinline__ void do_gateup(const SmallParams& p, const SmemPtrs& s, const SlotMeta& m,
                                          const uint8_t* slot, int tid, uint64_t* empty) {
    constexpr int V = kRowBatch * TM;
    const int uc = m.uc;  // the unit's ordinal in this CTA
    const int buf = uc & 1;
    constexpr int SHIFT = 5 - Log2<V>::value;
    const int warp = tid >> 5, lane = tid & 31;
    const SmallGeom& g = p.g;
    const int nb = p.H / 32;
    const int half = warp & 1, q = warp >> 1;
    const int c = half * 32 + lane;
    const int64_t rbH = (int64_t)p.H * WBITS / 8;
    const int rpg = 2 * g.rg / kRowGroups;  // rows per group: gate rows 0..rg-1, then up rows
    const int first = m.row0 - m.blk * kUnit;  // first pair of the chunk inside its unit
    const float* sg = reinterpret_cast<const float*>(slot + m.off_a);
    const float* su = reinterpret_cast<const float*>(slot + m.off_b);
    // the partials buffer of this unit was last read by the finisher of unit
    // uc - 2 (every chunk checks: with two groups a unit's chunks are split)
    if (uc >= 2 && !mbar_wait_ns(&s.ufree[buf], ((uc >> 1) - 1) & 1, kSlackWaits * p.wait_ns))
        set_error(p.err, kErrTimeout);
    // Branch-free inner loops (so that the independent dots interleave):
    // out-of-range blocks are clamped and get a zero scale, out-of-range rows
    // and tokens are clamped and their sums are never stored.
    const int nlast = m.n > 0 ? m.n - 1 : 0;
    for (int rb = 0; rb < rpg; rb += kRowBatch) {
        float acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.0f;
        const uint8_t* rowp[kRowBatch];
#pragma unroll
        for (int rr = 0; rr < kRowBatch; ++rr) {
            const int r = min(q * rpg + rb + rr, q * rpg + rpg - 1);
            rowp[rr] = slot + (size_t)r * rbH;
        }
#pragma unroll
        for (int j = 0; j < kMaxGuBlocks; ++j) {
            const int bj = c + kColThreads * j;
            const bool okb = bj < nb;
            const int b = okb ? bj : 0;
            ActBlock a[TM];
            float dx[TM];
            int cr[TM];
#pragma unroll
            for (int i = 0; i < TM; ++i) {
                const int t = tok_at(m, i < nlast ? i : nlast);
                a[i] = act_natural(*reinterpret_cast<const uint4*>(s.xq + ((size_t)(t * 2 + 0) * nb + b) * 16),
                                   *reinterpret_cast<const uint4*>(s.xq + ((size_t)(t * 2 + 1) * nb + b) * 16));
                dx[i] = okb ? s.xd[t * nb + b] * dot_unscale<WBITS>() : 0.0f;
                cr[i] = act_corr<WBITS>(a[i]);
            }
#pragma unroll
            for (int rr = 0; rr < kRowBatch; ++rr) {
                const WBlock<WBITS> w = load_block_smem<WBITS>(rowp[rr], b);
#pragma unroll
                for (int i = 0; i < TM; ++i)
                    acc[rr * TM + i] = fmaf(dx[i], (float)dot_block_scaled<WBITS>(w, a[i], cr[i]), acc[rr * TM + i]);
            }
        }
        const float v = warp_reduce_many<V>(acc, lane);
        const int vi = lane >> SHIFT;
        const int rr = vi / TM, i = vi % TM;
        if ((lane & ((1 << SHIFT) - 1)) == 0 && rb + rr < rpg && i < m.n) {
            const int r = q * rpg + rb + rr;
            const int gu = r < g.rg ? 0 : 1;
            const int up = first + (gu ? r - g.rg : r);
            s.gpart[(((buf * kUnit + up) * 2 + gu) * 2 + half) * 4 + i] = v;
        }
        if (half == 0 && lane < kRowBatch && rb + lane < rpg) {
            const int r = q * rpg + rb + lane;
            const int gu = r < g.rg ? 0 : 1;
            const int up = first + (gu ? r - g.rg : r);
            s.usc[(buf * kUnit + up) * 2 + gu] = gu ? su[r - g.rg] : sg[r];
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty);
    // Every warp reports each chunk's partials and goes on (the unit's first
    // chunk also leaves the unit's record); once all chunks of the unit are
    // in, the finisher warp turns them into h codes and publishes them
    if (first == 0 && warp == 0 && lane == 0) s.urec[buf] = UnitRec{m.entry, m.blk, m.slot0, m.n};
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.ufull[buf]);
}

// ---- the finisher warp: for each gate/up unit of the CTA (in order), wait
// until every consumer warp has reported its partials, then h = silu(g) * u
// for the 32 rows (lane = row) of each token, Q8_0 of the block, and the
// release of the codes to the other CTAs; the consumer warps never wait for
// this (nor for the release fence) ----
__device__ __forceinline__ void finisher(const SmallParams& p, const SmemPtrs& s, int lane) {
    bool open = false;  // the router barrier has completed (every CTA has read its counters)
    bool gave_up = false;
#pragma unroll 1
    for (int k = 0;; ++k) {
        const int buf = k & 1;
        if (!mbar_wait_ns(&s.ufull[buf], (k >> 1) & 1, kSlackWaits * p.wait_ns)) {
            if (lane == 0) set_error(p.err, kErrTimeout);
            return;
        }
        const UnitRec r = s.urec[buf];
        if (r.entry < 0) return;
        const float* gp = s.gpart + (buf * kUnit + lane) * 16;  // [gate/up][half][token]
        const float sgl = s.usc[(buf * kUnit + lane) * 2], sul = s.usc[(buf * kUnit + lane) * 2 + 1];
        const int n = r.n < 4 ? r.n : 4;
#pragma unroll 1
        for (int i = 0; i < n; ++i) {
            const float gs = gp[i] + gp[4 + i];
            const float us = gp[8 + i] + gp[12 + i];
            const float h = silu_mul(sgl * gs, sul * us);
            int8_t qv;
            float d;
            q8_0_warp(h, qv, d);
            const int64_t sl = r.slot0 + i;
            p.hq[sl * p.I + r.blk * kUnit + lane] = qv;
            if (lane == 0) p.hd[sl * (p.I / 32) + r.blk] = d;
        }
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&s.ufree[buf]);
            if (!open && !gave_up) {
                open = s.misc[9] && router_barrier_wait(p, s, kSlackWaits * p.wait_ns);
                gave_up = !open;
                if (gave_up && s.misc[9]) set_error(p.err, kErrTimeout);
            }
            fence_acq_rel_gpu();  // the warp's h codes before the count (release pattern)
            if (open && (r.entry != p.fault_entry || r.blk != 0)) red_add_relaxed_gpu(p.ctrl + kFcDone + r.entry, n);
        }
        open = __shfl_sync(kFull, open, 0);
        __syncwarp();
    }
}

// Activation block b of the down chunk's h codes (natural order in the slot)
// for every token, in the weights' order; blocks past the end get zero scale.
template <int WBITS, int TM>
__device__ __forceinline__ void down_act(const uint8_t* act, const float* hdv, int I, int nbI, int n, int bj,
                                         ActBlock (&a)[TM], float (&dh)[TM], int (&cr)[TM]) {
    const bool okb = bj < nbI;
    const int b = okb ? bj : 0;
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const int ii = i < n ? i : 0;
        const uint4 lo = *reinterpret_cast<const uint4*>(act + (size_t)ii * I + 32 * b);
        const uint4 hi = *reinterpret_cast<const uint4*>(act + (size_t)ii * I + 32 * b + 16);
        if constexpr (WBITS == 4) a[i] = act_nibble_order(lo, hi);
        else if constexpr (WBITS == 2) a[i] = act_crumb_order(lo, hi);
        else a[i] = act_natural(lo, hi);
        dh[i] = okb ? hdv[ii * nbI + b] * dot_unscale<WBITS>() : 0.0f;
        cr[i] = act_corr<WBITS>(a[i]);
    }
}

// ---- down chunk: nrows rows of Wd for the entry's tokens -> y ----
// Rows are dealt to the row groups round-robin (r = q + 4 k); the half-1
// warp of a pair hands its sums to the half-0 warp through shared memory.
template <int WBITS, int TM>
__device__ __forceinline__ void do_down(const SmallParams& p, const SmemPtrs& s, const SlotMeta& m,
                                        const uint8_t* slot, int tid, uint64_t* empty) {
    constexpr int RB = TM == 1 ? 16 : TM == 2 ? 8 : 4;  // rows of a group reduced together (all at decode)
    constexpr int V = RB * TM;
    constexpr int SHIFT = 5 - Log2<V>::value;
    const int warp = tid >> 5, lane = tid & 31;
    const int nbI = p.I / 32;
    const int half = warp & 1, q = warp >> 1;
    const int c = half * 32 + lane;
    const int64_t rbI = (int64_t)p.I * WBITS / 8;
    const uint8_t* act = slot + kSlotWeightBytes;
    const float* hdv = reinterpret_cast<const float*>(slot + m.off_a);
    const float* sdv = reinterpret_cast<const float*>(slot + m.off_b);
    // branch-free inner loops, as in the gate/up chunk; column block 0 of
    // the thread is loaded once, further ones (inter > 2048) per row batch
    const int nbj = (nbI + kColThreads - 1) / kColThreads;
    ActBlock a0[TM];
    float dh0[TM];
    int cr0[TM];
    const int b0 = c < nbI ? c : 0;
    down_act<WBITS, TM>(act, hdv, p.I, nbI, m.n, c, a0, dh0, cr0);
    const int nk = (m.nrows - q + kRowGroups - 1) / kRowGroups;  // rows of this group
    const int klast = nk > 0 ? nk - 1 : 0;
    for (int kb = 0; kb < nk; kb += RB) {
        float acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.0f;
        // sub-batches of 4 rows; one wholly past the group's rows is skipped
        // (a uniform branch), so a group of 10-11 rows computes 12
#pragma unroll
        for (int sb = 0; sb < RB / 4; ++sb) {
            if (kb + 4 * sb < nk) {
                const uint8_t* rowp[4];
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const int k = kb + 4 * sb + rr < klast ? kb + 4 * sb + rr : klast;
                    rowp[rr] = slot + (size_t)(q + kRowGroups * k) * rbI;
                }
#pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const WBlock<WBITS> w = load_block_smem<WBITS>(rowp[rr], b0);
#pragma unroll
                    for (int i = 0; i < TM; ++i)
                        acc[(4 * sb + rr) * TM + i] =
                            fmaf(dh0[i], (float)dot_block_scaled<WBITS>(w, a0[i], cr0[i]), acc[(4 * sb + rr) * TM + i]);
                }
                for (int j = 1; j < nbj; ++j) {
                    ActBlock aj[TM];
                    float dhj[TM];
                    int crj[TM];
                    const int bj = c + kColThreads * j;
                    down_act<WBITS, TM>(act, hdv, p.I, nbI, m.n, bj, aj, dhj, crj);
                    const int bc = bj < nbI ? bj : 0;
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        const WBlock<WBITS> w = load_block_smem<WBITS>(rowp[rr], bc);
#pragma unroll
                        for (int i = 0; i < TM; ++i)
                            acc[(4 * sb + rr) * TM + i] =
                                fmaf(dhj[i], (float)dot_block_scaled<WBITS>(w, aj[i], crj[i]), acc[(4 * sb + rr) * TM + i]);
                    }
                }
            }
        }
        const float v = warp_reduce_many<V>(acc, lane);
        const int vi = lane >> SHIFT;
        const int rr = vi / TM, i = vi % TM;
        const int r = q + kRowGroups * (kb + rr);
        if ((lane & ((1 << SHIFT) - 1)) == 0 && kb + rr < nk && i < m.n)
            s.ys[((m.slot0 + i) * p.g.rpc + m.blk + r) * 2 + half] = sdv[r] * v;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty);
}

// ---- COMBINE: the CTA's output rows from its per-slot down outputs (the
// two column halves of each row are added here, half 0 + half 1) ----
// ---- SYNC (two groups): this group's down outputs are all in ys (its
// items are processed in order); the other group's COMBINE waits for it ----
__device__ __forceinline__ void do_sync(const SmemPtrs& s, int tid, uint64_t* empty) {
    __syncwarp();
    if ((tid & 31) == 0) {
        mbar_arrive(s.gsync);
        mbar_arrive(empty);
    }
}

__device__ __forceinline__ void do_combine(const SmallParams& p, const SmemPtrs& s, const SlotMeta& m, int tid,
                                           uint64_t* empty, int group, int groups) {
    group_sync(group);  // every warp of this group has its down outputs in ys
    if (groups > 1 && !mbar_wait_ns(s.gsync, 0, kSlackWaits * p.wait_ns)) {  // and the other group's
        set_error(p.err, kErrTimeout);
        __syncwarp();
        if ((tid & 31) == 0) mbar_arrive(empty);
        return;
    }
    const int rows = m.nrows, T = p.T, k = p.k, rpc = p.g.rpc;
    const float2* ys = reinterpret_cast<const float2*>(s.ys);
    for (int idx = tid; idx < T * rows; idx += kConsumers) {
        const int t = idx / rows, r = idx - t * rows;
        float acc = 0.0f;  // fixed order: slots 0..k-1, then the shared expert
        for (int j = 0; j < k; ++j) {
            const int sl = s.inv[t * k + j];
            if (sl < 0 || sl >= T * k) continue;  // dropped by the adaptive top-p
            const float2 h = ys[sl * rpc + r];
            acc = fmaf(s.selw[t * k + j], h.x + h.y, acc);
        }
        if (p.ns) {
            const float2 h = ys[(T * k + t) * rpc + r];
            acc += h.x + h.y;
        }
        p.out[(int64_t)t * p.H + m.row0 + r] = acc;
    }
    // the per-slot outputs of these rows, for inspection
    for (int idx = tid; idx < p.g.nys * rows; idx += kConsumers) {
        const int sl = idx / rows, r = idx - sl * rows;
        const float2 h = ys[sl * rpc + r];
        p.y[(int64_t)sl * p.H + m.row0 + r] = h.x + h.y;
    }
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(empty);
}

// Output rows [r0, r1) that CTA c owns in the down projection and combine.
// More than one token: an even split.  One token: the gate/up units go round
// robin (unit u to CTA u mod grid, the shared expert's first), so the CTAs
// stream different numbers of units after the routing; they own rows in
// inverse measure, so that every CTA spends about the same time (its gate/up
// units + its rows of every entry's down matrix), as far as the row cap
// allows.  A shared-expert unit counts kSharedUnitCost of a routed one: its
// copies are issued before the routing and have landed when the consumers
// reach it, which they do while the routed experts' first copies are in
// flight (measured: weights 0, 0.3 and 0.6 gave 40.3, 40.55 and 40.6 us per
// decode step).  A down byte counts kDownCost times a gate/up byte (measured
// per SM, down chunks stream at about two thirds of the gate/up chunks' rate).
// With m = units - 1 = Q grid + rho and n_pre shared units (n_pre <= grid),
// the CTAs fall into four contiguous classes:
//   [0, min(n_pre, rho + 1))        Q routed units, one shared
//   [.., n_pre)                     Q - 1 routed, one shared
//   [n_pre, rho + 1)                Q + 1 routed
//   [max(n_pre, rho + 1), grid)     Q routed
// and a CTA of class X owns clamp((tt - w_X) unit_rows, 0, cap) rows, w_X its
// units, tt the common finish time that makes the rows add up to H (found
// on the host, own_tt).  Every CTA computes the same split.
struct OwnSplit {
    int lo[5];  // class X is CTAs [lo[X], lo[X + 1])
    double w[4], unit_rows, cap;
    bool even;  // an even split instead
    __host__ __device__ OwnSplit(int H, int I, int nu, int ns, int T, int grid, int rpc, int rd, int n_entries) {
        const int n_pre = ns ? nu : 0, n_all = n_entries * nu;
        even = T > 1 || n_entries <= 0 || n_pre > grid || n_all <= n_pre;
        const int Q = n_all > 0 ? (n_all - 1) / grid : 0, rho = n_all > 0 ? (n_all - 1) - Q * grid : 0;
        lo[0] = 0;
        lo[1] = n_pre < rho + 1 ? n_pre : rho + 1;
        lo[2] = n_pre;
        lo[3] = n_pre > rho + 1 ? n_pre : rho + 1;
        lo[4] = grid;
        w[0] = Q + kSharedUnitCost;
        w[1] = Q - 1 + kSharedUnitCost;
        w[2] = Q + 1;
        w[3] = Q;
        unit_rows = n_entries > 0 ? (double)(2 * kUnit * H) / (double)(n_entries * I) / kDownCost : 0.0;
        cap = (double)(rpc < rd ? rpc : rd);  // one down chunk per entry at most
        if (cap * grid < (double)H) even = true;  // the cap binds everywhere
    }
    // products and sums rounded one by one, in the same order on the host
    // (the table, the test export) and in every CTA
    static __host__ __device__ double mul(double a, double b) {
#ifdef __CUDA_ARCH__
        return __dmul_rn(a, b);
#else
        return a * b;
#endif
    }
    static __host__ __device__ double add(double a, double b) {
#ifdef __CUDA_ARCH__
        return __dadd_rn(a, b);
#else
        return a + b;
#endif
    }
    __host__ __device__ double rows_of(int x, double tt) const {
        const double r = mul(add(tt, -w[x]), unit_rows);
        return r < 0.0 ? 0.0 : (r > cap ? cap : r);
    }
    __host__ __device__ double prefix(int cc, double tt) const {  // rows of CTAs [0, cc)
        double v = 0.0;
        for (int x = 0; x < 4; ++x) {
            const int hi = cc < lo[x + 1] ? cc : lo[x + 1];
            if (hi > lo[x]) v = add(v, mul((double)(hi - lo[x]), rows_of(x, tt)));
        }
        return v;
    }
    // first row of CTA cc (grid: H)
    __host__ __device__ int start(int cc, int grid, int H, double tt) const {
        if (cc >= grid) return H;
        const int r = (int)floor(add(prefix(cc, tt), 1e-6));
        return r < H ? r : H;
    }
};

// The common finish time of the split (host; bisection to well below a row).
static double own_split_tt(const OwnSplit& o, int H, int grid) {
    if (o.even) return 0.0;
    double t0 = o.w[1] - 1.0, t1 = o.w[2] + 1.0 + (o.unit_rows > 0.0 ? (double)H / o.unit_rows : 0.0);
    for (int it = 0; it < 60; ++it) {
        const double tm = 0.5 * (t0 + t1);
        if (o.prefix(grid, tm) < (double)H) t0 = tm;
        else t1 = tm;
    }
    return t1;
}

__device__ __forceinline__ void owned_rows(const SmallParams& p, int n_entries, int c, int grid, int& r0, int& r1) {
    const int H = p.H;
    const OwnSplit o(H, p.I, p.g.nu, p.ns, p.T, grid, p.g.rpc, p.g.rd, n_entries);
    if (o.even || n_entries >= kOwnTab) {
        r0 = (int)((int64_t)H * c / grid);
        r1 = (int)((int64_t)H * (c + 1) / grid);
        return;
    }
    const double tt = p.own_tt[n_entries];
    r0 = o.start(c, grid, H, tt);
    r1 = o.start(c + 1, grid, H, tt);
}

// ---------------------------------------------------------------------------
// Main kernel
// ---------------------------------------------------------------------------
template <int WBITS, int TM>
__global__ void __launch_bounds__(Roles<TM>::kThreads, 1) k_moe_small(const __grid_constant__ SmallParams p) {
    using R = Roles<TM>;
    constexpr int G = R::kGroups;
    extern __shared__ __align__(128) uint8_t smem_raw[];
    const SmemPtrs s = carve(smem_raw, p.g);
    const SmallGeom& g = p.g;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int c = blockIdx.x, grid = gridDim.x;
    if (tid == 0) {
        for (int i = 0; i < g.nslot; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], kConsumerWarps);
        }
        mbar_init(s.routing, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.ufull[i], kConsumerWarps * g.cpu);  // every warp, every chunk of a unit
            mbar_init(&s.ufree[i], 1);
        }
        mbar_init(s.gsync, kConsumerWarps);
        mbar_init(s.gexit, G * kConsumerWarps);
        mbar_init(s.rowsin, 1);
        mbar_init(s.ctrl, 1);
        mbar_init(s.xqin, kConsumerWarps);
        fence_barrier_init();
    }
    // warp 0 reads the control region now (the values are stored to shared
    // memory later, by consumers_start, before this CTA's router arrival)
    CtrlSnap snap{};
    if (warp == 0) snap = ctrl_load(p, lane, g.nent);
    __syncthreads();

    if (warp == R::kFinisherWarp) {
        finisher(p, s, lane);
        return;
    }
    if (warp == R::kProducerWarp) {
        // ------------------------- producer -------------------------
        Producer pr(p, s, lane, G);
        const int64_t rowI = (int64_t)p.I * p.wbits / 8;
        // the CTA's router rows first (the selection waits for them), into
        // slot 0, which the selection's marker holds until it is done
        const int n_slot = router_rows_in_slot(p, c, grid);
        if (lane == 0) bulk_prefetch_l2(p.x, (uint32_t)(p.T * p.H * 4));  // x ahead of every copy
        if (n_slot > 0 && lane == 0) {
            mbar_arrive_expect_tx(s.rowsin, (uint32_t)(n_slot * p.H * 4));
            for (int i = 0; i < n_slot; ++i)
                bulk_g2s_nohint(s.slots + (size_t)i * p.H * 4, p.router_w + (int64_t)(c + grid * i) * p.H,
                                (uint32_t)(p.H * 4), s.rowsin);
        }
        pr.marker(kItemSelect);
        {
            // the shared expert's down rows this CTA will probably own
            int q0, q1;
            owned_rows(p, p.k + (p.ns ? 1 : 0), c, grid, q0, q1);
            if (p.ns && lane == 0 && q1 > q0)
                bulk_prefetch_l2(p.shared.w_down + (int64_t)q0 * rowI, (uint32_t)((q1 - q0) * rowI));
        }
        // the shared expert's gate/up units need no routing
        EntryInfo e0;
        e0.expert = -1;
        e0.slot0 = p.T * p.k;
        e0.n = p.T;
        for (int i = 0; i < 4; ++i) e0.tok[i] = i < p.T ? i : 0;
        const int n_pre = p.ns ? g.nu : 0;
        for (int u = c; u < n_pre; u += grid)
            for (int ch = 0; ch < g.cpu; ++ch) pr.gateup(0, e0, u, ch);
        // the routed part of the schedule needs this CTA's routing tables
        int ok = 1;
        if (lane == 0) ok = mbar_wait_ns(s.routing, 0, kSlackWaits * p.wait_ns) ? 1 : 0;
        ok = __shfl_sync(kFull, ok, 0);
        __syncwarp();  // lane 0's acquire of the tables orders the other lanes' reads
        if (!ok) pr.fail();
        if (!s.misc[9]) pr.aborted = true;  // uninitialised control region: no routed work (error recorded)
        const int umax = g.nent - 1;
        int U = s.misc[0];
        U = U < 0 ? 0 : (U > umax ? umax : U);
        const int first = p.ns ? 0 : 1;
        const int n_routed = U * g.nu;
        if (p.T > 1) {
            // the routed experts' units are taken from a global counter, one
            // at a time (requested one unit ahead): SMs that stream faster
            // take more, so every CTA reaches its down chunks at about the
            // same time
            int next = 0;
            if (lane == 0) next = (int)((uint32_t)atom_add_relaxed_gpu(p.ctrl + kFcUnits, 1) - s.base[0]);
            next = __shfl_sync(kFull, next, 0);
            while (next < n_routed && !pr.aborted) {
                const int r = next;
                if (lane == 0) next = (int)((uint32_t)atom_add_relaxed_gpu(p.ctrl + kFcUnits, 1) - s.base[0]);
                const int entry = 1 + r / g.nu, blk = r % g.nu;
                const EntryInfo ei = s.ent[entry];
                for (int ch = 0; ch < g.cpu; ++ch) pr.gateup(entry, ei, blk, ch);
                next = __shfl_sync(kFull, next, 0);
            }
        } else {
            // one token: a static round robin over the units of all experts
            // (the shared expert's first, issued above) measured as fast
            const int n_pre_all = p.ns ? g.nu : 0;
            for (int u = c; u < n_pre_all + n_routed && !pr.aborted; u += grid) {
                if (u < n_pre_all) continue;
                // before the CTA's last unit: one poll of the entries' h
                // counters, so that the first down chunks (of entries that
                // completed in the earlier rounds) follow it without a round
                // trip (the producer would wait for a ring slot meanwhile)
                if (u + grid >= n_pre_all + n_routed) pr.poll_entries(U);
                const int entry = 1 + (u - n_pre_all) / g.nu, blk = (u - n_pre_all) % g.nu;
                const EntryInfo ei = s.ent[entry];
                for (int ch = 0; ch < g.cpu; ++ch) pr.gateup(entry, ei, blk, ch);
            }
        }
        int r0, r1;
        owned_rows(p, U + (p.ns ? 1 : 0), c, grid, r0, r1);
        for (int entry = first; entry <= U && !pr.aborted; ++entry) {
            const EntryInfo ei = s.ent[entry];
            for (int rr = r0; rr < r1; rr += g.rd) {
                if (!pr.wait_entry(entry, U)) break;
                pr.down(entry, ei, rr, (r1 - rr) < g.rd ? (r1 - rr) : g.rd, rr - r0);
            }
        }
        if (!pr.aborted) {
            // two groups: the SYNC marker goes to one group, the COMBINE
            // marker (the next slot) to the other, which waits for it
            if (G > 1) pr.marker(kItemSync);
            SlotMeta m = pr.blank(kItemCombine);
            m.row0 = r0;
            m.nrows = r1 - r0;
            pr.push(m, no_copy(), no_copy(), no_copy(), no_copy());
        }
        pr.finish();  // a DONE marker per group
        pr.drain();
        return;
    }

    // ------------------------- consumers -------------------------
    const int group = warp / kConsumerWarps;     // consumer group
    const int gtid = tid - group * kConsumers;   // thread index inside the group
    consumers_start<WBITS, TM>(p, s, s.slots, snap, tid, G * kConsumers);
    // group g takes ring slots g, g + G, ... in order
    int slot = group;
    uint32_t pf = 0;
    int units = 0;  // the CTA's gate/up units, from the DONE marker (or the last unit seen)
    bool xq_staged = false;
    while (true) {
        if (!mbar_wait_ns(&s.full[slot], pf, kSlackWaits * p.wait_ns)) {
            set_error(p.err, kErrTimeout);
            break;
        }
        const SlotMeta m = s.meta[slot];
        uint8_t* data = s.slots + (size_t)slot * g.slot_bytes;
        uint64_t* empty = &s.empty[slot];
        if (m.kind == kItemGateUp) {
            if (!xq_staged) {  // the first gate/up item: the selecting group has staged xq
                int okx = 1;
                if (lane == 0) okx = mbar_wait_ns(s.xqin, 0, kSlackWaits * p.wait_ns) ? 1 : 0;
                if (!__shfl_sync(kFull, okx, 0) && lane == 0) set_error(p.err, kErrTimeout);
                __syncwarp();  // lane 0's acquire orders the other lanes' reads
                xq_staged = true;
            }
            // the loops are unrolled over the entry's own token count (an
            // entry with fewer tokens than the batch does not compute the
            // clamped copies)
            if (TM == 1 || m.n <= 1) do_gateup<WBITS, 1>(p, s, m, data, gtid, empty);
            else if (TM == 2 || m.n == 2) do_gateup<WBITS, TM == 1 ? 1 : 2>(p, s, m, data, gtid, empty);
            else do_gateup<WBITS, TM>(p, s, m, data, gtid, empty);
            units = max(units, m.uc + 1);
        } else if (m.kind == kItemDown) {
            if (TM == 1 || m.n <= 1) do_down<WBITS, 1>(p, s, m, data, gtid, empty);
            else if (TM == 2 || m.n == 2) do_down<WBITS, TM == 1 ? 1 : 2>(p, s, m, data, gtid, empty);
            else do_down<WBITS, TM>(p, s, m, data, gtid, empty);
        } else if (m.kind == kItemSelect) {
            // always group 0's: the first item; every CTA's logits first
            if (s.misc[9]) {
                if (gtid == 0 && !router_barrier_wait(p, s, kSlackWaits * p.wait_ns)) set_error(p.err, kErrTimeout);
                consumers_sync();
                do_select(p, s, data, gtid);
            } else if (gtid == 0) {  // no routing: the producer winds down
                s.misc[0] = 0;
                s.misc[1] = 0;
                mbar_arrive(s.routing);
            }
            // every CTA's share of xq is published (the router barrier), and
            // the producer is already streaming the routed experts: their
            // latency covers this staging
            {
                XqStage<WBITS, TM> xs;
                xs.load(p, gtid);
                xs.store(p, s, gtid);
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(s.xqin);
                mbar_arrive(empty);  // the slot was the scratch
            }
        } else if (m.kind == kItemSync) {
            do_sync(s, gtid, empty);
        } else if (m.kind == kItemCombine) {
            do_combine(p, s, m, gtid, empty, group, G);
        } else {
            if (m.kind == kItemDone) units = m.uc;
            break;  // DONE (or an unknown marker)
        }
        slot += G;
        if (slot >= g.nslot) {
            slot = group;
            pf ^= 1u;
        }
    }
    // No more units: once every consumer warp has left its loop, hand the
    // finisher a terminal record with the full arrival count (its buffer was
    // last used by unit units - 2, which the finisher must have read first).
    if (gtid == 0) s.misc[4 + group] = units;
    __syncwarp();
    if (lane == 0) mbar_arrive(s.gexit);
    if (tid == 0) {
        bool ok = mbar_wait_ns(s.gexit, 0, kSlackWaits * p.wait_ns);
        int n = s.misc[4];
        for (int gi = 1; gi < G; ++gi) n = max(n, s.misc[4 + gi]);
        const int buf = n & 1;
        if (ok && n >= 2) ok = mbar_wait_ns(&s.ufree[buf], ((n >> 1) - 1) & 1, kSlackWaits * p.wait_ns);
        if (!ok) set_error(p.err, kErrTimeout);
        s.urec[buf] = UnitRec{-1, 0, 0, 0};
        mbar_arrive_count(&s.ufull[buf], (uint32_t)(kConsumerWarps * g.cpu));
    }
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------
// The persistent kernel's CTAs wait for one another (the down chunks wait for
// other CTAs' h codes), so the grid must be resident all at once: it is
// launched as a cooperative grid (one CTA per SM), which the runtime only
// starts when every CTA can run, also beside another forward on another
// stream.
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
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_moe_small<WBITS, TM>, Roles<TM>::kThreads,
                                                          prm.g.smem_bytes);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        attr_done[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prm.g.grid);
    cfg.blockDim = dim3(Roles<TM>::kThreads);
    cfg.dynamicSmemBytes = prm.g.smem_bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_moe_small<WBITS, TM>, prm);
}

// The one-token down-row split of a grid, as every CTA computes it (test
// export): starts[c] = the first row of CTA c, starts[grid] = hidden.
int small_down_rows(const moe_config& c, int T, int n_entries, int grid, int32_t* starts) {
    const SmallGeom g = small_geometry(c, T, grid);
    const OwnSplit o(c.hidden, c.inter, g.nu, c.n_shared, T, grid, g.rpc, g.rd, n_entries);
    if (o.even || n_entries >= kOwnTab) {
        for (int cc = 0; cc <= grid; ++cc) starts[cc] = (int32_t)((int64_t)c.hidden * cc / grid);
        return 0;
    }
    const double tt = own_split_tt(o, c.hidden, grid);
    for (int cc = 0; cc <= grid; ++cc) starts[cc] = o.start(cc, grid, c.hidden, tt);
    return (int)o.cap;
}

// Test hook state (moe_debug_fault_injection): read by every launch.
static std::atomic<int> g_fault_entry{-1};
static std::atomic<long long> g_wait_ns{(long long)kWaitNs};

void set_fault_injection(int withhold_entry, int64_t wait_ns) {
    g_fault_entry.store(withhold_entry < 0 ? -1 : withhold_entry);
    g_wait_ns.store(wait_ns > 0 ? (long long)wait_ns : (long long)kWaitNs);
}

cudaError_t launch_small(const SmallArgs& a, cudaStream_t st) {
    const moe_config& c = *a.cfg;
    SmallParams p;
    p.T = a.T; p.H = c.hidden; p.I = c.inter; p.E = c.n_experts; p.G = c.n_groups; p.tg = c.topk_groups;
    p.k = c.top_k; p.ns = c.n_shared; p.wbits = c.wbits; p.rsf = c.routed_scaling_factor; p.topp = c.expert_topp;
    p.ep_lo = a.ep_lo; p.ep_hi = a.ep_hi;
    p.x = a.x; p.router_w = a.router_w; p.bias = a.bias; p.routed = a.routed; p.shared = a.shared;
    p.xq = a.xq; p.xd = a.xd; p.logits = a.logits; p.idx = a.idx; p.w = a.w; p.counts = a.counts;
    p.offsets = a.offsets; p.perm = a.perm; p.inv_perm = a.inv_perm; p.active = a.active;
    p.hq = a.hq; p.hd = a.hd; p.y = a.y; p.out = a.out; p.ctrl = a.ctrl; p.err = a.err;
    p.wait_ns = (uint64_t)g_wait_ns.load();
    p.fault_entry = g_fault_entry.load();
    p.rows_bulk = (reinterpret_cast<uintptr_t>(a.router_w) % 16 == 0) ? 1 : 0;
    p.g = small_geometry(c, a.T, device_info().sm_count);
    {
        // the down-row split's finish times, per entry count (one token);
        // recomputed only when the split's inputs change
        static std::mutex mu;
        static int key[8] = {-1, -1, -1, -1, -1, -1, -1, -1};
        static double tab[kOwnTab];
        const int k8[8] = {p.H, p.I, p.g.nu, p.ns, a.T == 1 ? 1 : 2, p.g.grid, p.g.rpc, p.g.rd};
        std::lock_guard<std::mutex> lock(mu);
        if (!std::equal(k8, k8 + 8, key)) {
            for (int n = 0; n < kOwnTab; ++n) {
                const OwnSplit o(p.H, p.I, p.g.nu, p.ns, a.T, p.g.grid, p.g.rpc, p.g.rd, n);
                tab[n] = own_split_tt(o, p.H, p.g.grid);
            }
            std::copy(k8, k8 + 8, key);
        }
        std::copy(tab, tab + kOwnTab, p.own_tt);
    }
    if (p.g.smem_bytes > device_info().max_smem_optin) return cudaErrorInvalidConfiguration;
    const int tm = p.g.tmax;
    if (c.wbits == 4) {
        if (tm == 1) return launch_small_t<4, 1>(p, st);
        if (tm == 2) return launch_small_t<4, 2>(p, st);
        return launch_small_t<4, 4>(p, st);
    }
    if (c.wbits == 2) {
        if (tm == 1) return launch_small_t<2, 1>(p, st);
        if (tm == 2) return launch_small_t<2, 2>(p, st);
        return launch_small_t<2, 4>(p, st);
    }
    if (tm == 1) return launch_small_t<8, 1>(p, st);
    if (tm == 2) return launch_small_t<8, 2>(p, st);
    return launch_small_t<8, 4>(p, st);
}

}  // namespace moe
