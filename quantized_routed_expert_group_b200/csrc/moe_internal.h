// moe_internal.h -- launchers and workspace layout shared by the library's
// translation units (not part of the public ABI).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

// Workspace regions for a call with T tokens.  Every region starts on a
// 256-byte boundary.  "slots" = T*top_k routed pairs + T*n_shared shared.
struct Layout {
    size_t err;        // int32[16]: [0] error word, [1..] counters
    size_t xin;        // fp32 [T][H]  host-copied activations (forward_host)
    size_t outbuf;     // fp32 [T][H]  result staged for the host copy
    size_t xq;         // int8 [T][H]
    size_t xd;         // fp32 [T][H/32]
    size_t logits;     // fp64 [T][E]
    size_t idx;        // int32 [T][k]
    size_t idx_ep;     // int32 [T][k]  idx with the picks outside this call's expert range as -1
    size_t w;          // fp32 [T][k]
    size_t counts;     // int32 [E]
    size_t offsets;    // int32 [E+1]
    size_t perm;       // int32 [T*k]
    size_t inv_perm;   // int32 [T*k]
    size_t active;     // int32 [1 + E + 1]: count, then expert ids
    size_t ctrl;       // int32 control words of the fused small-batch kernel
    size_t hbuf;       // fp32 [slots][I]  h before quantisation (fused kernel)
    size_t hq;         // int8 [slots][I]
    size_t hd;         // fp32 [slots][I/32]
    size_t y;          // fp32 [slots][H]
    // batched tensor-core path only (0 bytes otherwise)
    size_t tc_xg, tc_xdT, tc_gu, tc_hg, tc_hdT, tc_row_tok, tc_row_slot, tc_units_gu, tc_units_dn, tc_ctrl;
    size_t tc_xp, tc_hp, tc_pex, tc_peh, tc_xpt, tc_pet;
    size_t total;
};

Layout make_layout(const moe_config& c, int T);

// Record a tracing event on s.  Inside a stream capture a plain record only
// orders the graph; an external record makes the graph record the event when
// it runs, so the phase events time captured forwards too.
inline cudaError_t record_event(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const cudaError_t e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return e;
    return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
                                               : cudaEventRecord(ev, s);
}

struct DeviceInfo {
    int sm_count;
    int max_smem_optin;
};
const DeviceInfo& device_info();

// ---- launchers (return cudaError_t of the launch) ----
cudaError_t launch_quantize_q8_0(const float* x, int64_t n_rows, int cols, int8_t* q, float* d,
                                 cudaStream_t s);
cudaError_t launch_pack_weights(const float* w, int64_t rows, int cols, int wbits, uint8_t* packed,
                                float* scales, cudaStream_t s);
cudaError_t launch_requant_fp8(const uint8_t* w8, const float* block_scales, int64_t rows, int cols, int block,
                               int wbits, uint8_t* packed, float* scales, cudaStream_t s);
// The router's workspace: logits [T][E] fp64, then (T >= kRouterTiledMinTokens)
// the tiled kernel's K-split partial sums.
constexpr int kRouterTiledMinTokens = 5;  // below: the per-token kernel (the fused path's sizes)
size_t router_ws_bytes(const moe_config& c, int T);
cudaError_t launch_router(const moe_config& c, const float* x, int T, const float* router_w,
                          const float* bias, double* logits, int32_t* idx, float* w, cudaStream_t s);
// idx_ep = idx with every pick outside [lo, hi) replaced by -1.
cudaError_t launch_ep_mask(const int32_t* idx, int64_t n, int lo, int hi, int32_t* idx_ep, cudaStream_t s);
cudaError_t launch_bucket(const moe_config& c, const int32_t* idx, int T, int32_t* counts,
                          int32_t* offsets, int32_t* perm, int32_t* inv_perm, int32_t* active,
                          int32_t* err, cudaStream_t s);
size_t bucket_smem_bytes(const moe_config& c, int T);

struct ExpertArgs {
    const moe_config* cfg;
    int T;
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
// ev (optional, 3 events): recorded after gate/up, down and combine.
cudaError_t launch_experts(const ExpertArgs& a, cudaStream_t s, cudaEvent_t const* ev);
// The one-token down-row split (fused path) as every CTA computes it; returns
// the row cap, 0 for an even split (test export).
int small_down_rows(const moe_config& c, int T, int n_entries, int grid, int32_t* starts);
int router_splits(const moe_config& c, int T);
constexpr int kForwardLaunches = 7;  // quantise, logits, select, bucket, gate/up, down, combine
// (+1 when the router logits take the split-K form: router_splits > 0)
cudaError_t launch_combine(const ExpertArgs& a, cudaStream_t s);

// Batched path on the tensor cores (moe_tc.cu), for T >= kTcMinTokens.
constexpr int kTcMinTokens = 64;
// quantise (with the digit planes), router logits, their split-K reduce, select,
// bucket, plan, gather; gate/up on the digit planes and its fp64 fallback (one
// of the two returns at once), SwiGLU, down and its fallback, combine
constexpr int kTcLaunches = 13;
bool tc_path_supported(const moe_config& c, int T);
struct TcSizes {
    int prows_cap;     // rows of the padded row space
    int units_gu_cap;  // work units of the gate/up GEMM
    int units_dn_cap;  // work units of the down GEMM
};
TcSizes tc_sizes(const moe_config& c, int T);
struct TcArgs {
    ExpertArgs ex;
    int8_t* xg;         // [prows_cap][hidden]
    double* xdT;        // [hidden/32][prows_cap]
    float* gu;          // [2][prows_cap][inter]  g and u row values
    int8_t* hg;         // [prows_cap][inter]
    double* hdT;        // [inter/32][prows_cap]
    int8_t* xp;         // [prows_cap][5][hidden]  digit planes of the scaled x codes
    int8_t* hp;         // [prows_cap][5][inter]   digit planes of the scaled h codes
    double* pex;        // [prows_cap] 2^E of each row's x planes
    double* peh;        // [prows_cap] 2^E of each row's h planes
    int8_t* xpt;        // [T][5][hidden] digit planes of each token (k_tc_quantize)
    double* pet;        // [T] 2^E of each token's planes
    int* xwide;         // some token's block scales spread too far for the planes (zeroed per call)
    int* hwide;         // the same for some row of h
    int32_t* row_tok;   // [prows_cap]
    int32_t* row_slot;  // [prows_cap]
    void* units_gu;     // TcUnit [units_gu_cap]
    void* units_dn;     // TcUnit [units_dn_cap]
    int32_t* ctrl;      // [16]
    TcSizes sz;
};
constexpr size_t kTcUnitBytes = 16;
// Q8_0 of x and each token's digit planes (the batched path's quantiser)
cudaError_t launch_tc_quantize(const float* x, int T, int H, int8_t* xq, float* xd, int8_t* xpt, double* pet,
                               int* xwide, cudaStream_t s);
// plan + gather (the end of the bucketing phase)
cudaError_t launch_tc_prepare(const TcArgs& a, cudaStream_t s);
// gate/up GEMM, down GEMM, combine; ev (optional, 3 events) after each
cudaError_t launch_tc_experts(const TcArgs& a, cudaStream_t s, cudaEvent_t const* ev);
// Fused small-batch forward (T <= 4), moe_small.cu.
struct SmallArgs {
    const moe_config* cfg;
    int T;
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
    int32_t* err;
    int ep_lo, ep_hi;  // routed experts computed by this call: [ep_lo, ep_hi)
};
bool small_path_supported(const moe_config& c, int T);
// The fused path's control region: at a fixed workspace offset (the same
// for every T), kept from one call to the next; launch_fused_ctrl_init
// initialises it (zeros and a marker) before the first fused forward.
constexpr size_t kFusedCtrlBytes = 1024;
cudaError_t launch_fused_ctrl_init(int* ctrl, cudaStream_t s);
cudaError_t launch_small(const SmallArgs& a, cudaStream_t s);
constexpr int kSmallLaunches = 1;  // the persistent kernel
// Test hook (moe_debug_fault_injection): withhold one entry's first h
// publication in the fused kernel, and bound its producer waits by wait_ns
// (<= 0: the default).
void set_fault_injection(int withhold_entry, int64_t wait_ns);

cudaError_t launch_block_dots(const uint8_t* packed, int64_t rows, int cols, int wbits, const int8_t* q,
                              int n, int32_t* out, cudaStream_t s, int routine);
// Tensor-core per-block dots (moe_tc.cu): n <= 64 token rows of q.
cudaError_t launch_tc_block_dots(const uint8_t* packed, int64_t rows, int cols, int wbits, const int8_t* q, int n,
                                 int32_t* out, cudaStream_t s);
cudaError_t launch_synth_normal(uint64_t seed, uint64_t tid, int64_t offset, int64_t n, float sigma,
                                float* out, cudaStream_t s);

}  // namespace moe
