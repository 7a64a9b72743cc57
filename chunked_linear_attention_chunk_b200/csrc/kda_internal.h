// kda_internal.h -- host-side launch declarations shared by the libkda translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

int num_sms();  // SM count of the current device (cached per device)

// Device address of the current device's kernel status word (see kda_device_status).
unsigned int *device_status_ptr();

// K1: g = g_min * sigmoid(a), fp64-exact, n elements.
cudaError_t launch_gate(const void *a, kda_dtype dt, double g_min, float *g, int64_t n, cudaStream_t s);
cudaError_t launch_gate_heads(const void *a, kda_dtype dt, double g_min, const float *A_log, int64_t n_tok, int H,
                              int dk, float *g, cudaStream_t s);

// The gate of all 65536 bfloat16 inputs (per head with A_log, H x 65536 entries), from the
// same fp64 functions as the kernels above: the chunk kernels look g up in it.
constexpr size_t kGateTableEntries = 65536;
cudaError_t launch_gate_table(bool logsigmoid, double g_min, const float *A_log, int H, float *tab, cudaStream_t s);

// K5: float32 CUDA-core chunked forward (16-token chunks).
cudaError_t launch_chunk_f32(int B, int T, int H, int D, const float *q, const float *k, const float *v,
                             const float *a, const float *beta, float g_min, const float *S0, float *o,
                             float *S_T, cudaStream_t s);

// K2 + K3: bfloat16 tensor-core chunked forward.  The prep writes one record per (b*h,
// chunk) into the workspace; the scan walks them.  `logsigmoid` selects the unbounded gate
// g = log sigmoid(a) with element-wise diagonal tiles (g_min is then not used).  A_log
// (nullable, [H]) scales the gate's argument by e^{A_log[h]}.
// The workspace holds the records, then one gate table per head (the per-head scale needs
// them; without it only the first is written): chunk_bf16_records + H x 65536 floats.
size_t chunk_bf16_records(int B, int T, int H, int D);
size_t chunk_bf16_workspace(int B, int T, int H, int D);
cudaError_t launch_prep_bf16(int B, int T, int H, int D, const void *q, const void *k, const void *v,
                             const void *a, const void *beta, float g_min, bool logsigmoid, const float *A_log,
                             void *workspace, cudaStream_t s);
cudaError_t launch_scan_bf16(int B, int T, int H, int D, const void *workspace, const float *S0, void *o,
                             float *S_T, cudaStream_t s);

// Sequence-parallel pieces: the scan over one segment's records from S = 0 (S_zero) and of
// the identity without Bm (M, the segment's transfer map), and the prefix combine
// S_in[r + 1] = M[r] S_in[r] + S_zero[r] over R segments (dk == dv == D).
cudaError_t launch_scan_affine_bf16(int B, int T, int H, int D, const void *workspace, float *S_zero, float *M,
                                    cudaStream_t s);
cudaError_t launch_combine(int R, int BH, int D, const float *M, const float *S_zero, const float *S0, float *S_in,
                           cudaStream_t s);

// Packed variable-length batch: N sequences on one axis of T tokens, sequence s spanning
// [cu[s], cu[s+1]) (cu on the device).  A table kernel validates cu and writes the chunk
// offsets at the end of the workspace; prep and scan follow on the same stream.
size_t chunk_bf16_varlen_workspace(int N, int T, int H, int D);
cudaError_t launch_chunk_bf16_varlen(int N, const int32_t *cu, int T, int H, int D, const void *q, const void *k,
                                     const void *v, const void *a, const void *beta, float g_min, bool logsigmoid,
                                     const float *A_log, const float *S0, void *o, float *S_T, void *workspace,
                                     cudaStream_t s);

// Backward of the bf16 chunked forward (bounded gate, optional per-head scale A_log): prep,
// the scan saving every chunk's entering state, the reverse state-gradient scan, the
// per-chunk gradients and (with dA_log) the per-head reduction of dL/dA_log.  Gradients are
// float32; A_log, S0, dS_T, dS0 and dA_log are nullable.
size_t chunk_bf16_bwd_workspace(int B, int T, int H, int D);
void chunk_bf16_bwd_offsets(int B, int T, int H, int D, size_t *states, size_t *dstates);
cudaError_t launch_chunk_bwd_bf16(int B, int T, int H, int D, const void *q, const void *k, const void *v,
                                  const void *a, const void *beta, float g_min, const float *A_log, const float *S0,
                                  const void *dO, const float *dS_T, float *dq, float *dk, float *dv, float *da,
                                  float *dbeta, float *dS0, float *dA_log, void *workspace, cudaStream_t s,
                                  bool have_records = false);
// (have_records: the workspace already holds the records and gate table the forward's prep
// wrote for the same inputs, at the same offsets; the prep is not launched again.)
// The same over a packed batch (cu on the device, checked on the device as in the forward).
size_t chunk_bf16_bwd_varlen_workspace(int N, int T, int H, int D);
cudaError_t launch_chunk_bwd_bf16_varlen(int N, const int32_t *cu, int T, int H, int D, const void *q, const void *k,
                                         const void *v, const void *a, const void *beta, float g_min,
                                         const float *A_log, const float *S0, const void *dO, const float *dS_T,
                                         float *dq, float *dk, float *dv, float *da, float *dbeta, float *dS0,
                                         float *dA_log, void *workspace, cudaStream_t s);
// All checks of one kda_chunk_fwd problem, on the whole (B, T) problem at once; with
// check_ws false the workspace range is only used for the overlap checks (its size is the
// caller's business).  dispatch_chunk_fwd launches a problem that passed them.
kda_status validate_chunk_fwd(int B, int T, int H, int dk, int dv, kda_dtype dtype, const void *q, const void *k,
                              const void *v, const void *a, const void *beta, float g_min, kda_gate gate,
                              const float *S0, const void *o, const float *S_T, const void *workspace,
                              size_t ws_bytes, bool check_ws);
kda_status dispatch_chunk_fwd(int B, int T, int H, int dk, kda_dtype dtype, const void *q, const void *k,
                              const void *v, const void *a, const void *beta, float g_min, kda_gate gate,
                              const float *S0, void *o, float *S_T, void *workspace, cudaStream_t s);
// K4: single-token decode step.
cudaError_t launch_decode(int N, int H, int D, kda_dtype dt, const void *q, const void *k, const void *v,
                          const void *a, const void *beta, float g_min, float *S, void *o, cudaStream_t s);

}  // namespace kda
