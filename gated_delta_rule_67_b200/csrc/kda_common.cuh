// kda_common.cuh -- small helpers shared by the KDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// Element loads/stores for the two supported I/O types.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

struct WorkspaceHeader;

// Launch entry points implemented in the individual .cu files.  Arguments
// have been validated by the API layer.  Each returns the cudaError_t of its
// launch(es).
cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* g, const void* beta,
                          float scale, float* state, void* o, int N, int H, int dk, int dv, int dtype,
                          int gate, int prep, cudaStream_t stream);

cudaError_t launch_prefill_f32(const float* q, const float* k, const float* v, const float* g,
                               const float* beta, float scale, const float* s0, float* o, float* sT,
                               int B, int T, int H, int dk, int dv, int chunk, int gate, int prep,
                               cudaStream_t stream, void* const* events);

// bf16 chunked prefill (tcgen05 path).  `ws` is the caller's workspace.
size_t prefill_bf16_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk);
int prefill_bf16_launches(int B, int T, int H);
cudaError_t launch_prefill_bf16(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                const __nv_bfloat16* g, const __nv_bfloat16* beta, float scale,
                                const float* s0, __nv_bfloat16* o, float* sT, int B, int T, int H,
                                int dk, int dv, int chunk, int gate, int prep, void* ws, size_t ws_bytes,
                                cudaStream_t stream, void* const* events);

// The backward's tensor-core pass record (d_k = d_v = 128): 128-byte-swizzled
// token-row tiles, element (token i, channel c) of a [64][128] tile at byte
// (c / 64) * 8192 + i * 128 + (((c % 64) / 8) ^ (i % 8)) * 16 + (c % 8) * 2
// (A_qk: [64 query tokens][64 key tokens], one 8 KiB half).
constexpr uint32_t kTcRecW = 0, kTcRecQp = 16384, kTcRecKb = 32768, kTcRecAqk = 49152, kTcRecBytes = 57344;

// The per-chunk operands of the backward (bf16, d_k = d_v = 128, tensor-core
// state passes), written by the prefill's preparation kernel in its backward
// mode: record = (sequence, head) index within the launch group * NC + chunk.
struct PrepBwdOut {
  uint8_t* rec;       // pass records: W, Q+, Kbar, A_qk at the kTcRec* offsets
  size_t rec_stride;  // bytes between consecutive records
  float* P;           // [rec][64][64] strict_tril(K+ K-^T), fp32
  __nv_bfloat16* T;   // [rec][64][64] (I + diag(beta) P)^-1, bf16, row-major
  float* U;           // [rec][64][128] T diag(beta) V, fp32
  float* gam;         // [rec][128] exp(G_C)
  int bh0;            // (sequence, head) of the launch's first record
  int nbh;            // (sequence, head) pairs in the launch
};
cudaError_t launch_prep_for_backward(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                     const __nv_bfloat16* g, const __nv_bfloat16* beta, float scale, int B, int T,
                                     int H, int gate, const PrepBwdOut& out, struct WorkspaceHeader* hdr,
                                     cudaStream_t stream);

// Backward pass (kda_backward_chunk.cu).  The workspace holds a
// WorkspaceHeader (error word of the bounded waits; at the start of `ws`
// unless `hdr` points elsewhere) and the records of one or more (sequence,
// head) pairs; the pairs are processed in groups of as many as fit (at least
// backward_workspace_bytes(1, T, 1, dk, dv, dtype) bytes, header included).
size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype);
cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* g, const void* beta,
                            float scale, const float* s0, const void* d_o, const float* dsT, void* dq, void* dk_out,
                            void* dv_out, void* dg, void* dbeta, float* ds0, int B, int T, int H, int dk, int dv,
                            int dtype, int gate, void* ws, size_t ws_bytes, cudaStream_t stream,
                            float* dq32 = nullptr, float* dk32 = nullptr, struct WorkspaceHeader* hdr = nullptr);

// Backward through the fused input preparation (kda_backward_prep.cu): the
// workspace holds backward_prep_bytes of prepared inputs, then the records.
size_t backward_prep_bytes(int B, int T, int H, int dk, int dtype);
cudaError_t launch_backward_prepared(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                     float scale, const float* s0, const void* d_o, const float* dsT, void* dq,
                                     void* dk_out, void* dv_out, void* dg, void* dbeta, float* ds0, int B, int T, int H,
                                     int dk, int dv, int dtype, int gate, int prep, void* ws, size_t ws_bytes,
                                     cudaStream_t stream);

// Launches a kernel whose only wait can never be satisfied (short limit).
cudaError_t launch_wait_selftest(void* ws, cudaStream_t stream);

// Fused input preparation (kda_prep).
constexpr int kPrepMask = KDA_PREP_L2NORM_QK | KDA_PREP_GATE_LOGSIGMOID | KDA_PREP_BETA_SIGMOID;
constexpr float kL2Eps = 1e-6f;  // q <- q (sum q^2 + kL2Eps)^-1/2
__device__ __forceinline__ float log_sigmoid(float x) { return fminf(x, 0.f) - log1pf(expf(-fabsf(x))); }
__device__ __forceinline__ float sigmoidf(float x) { return 1.f / (1.f + expf(-x)); }
// Same with the fast exp/log intrinsics (absolute error ~1e-7; for bf16 inputs).
__device__ __forceinline__ float log_sigmoid_fast(float x) { return fminf(x, 0.f) - __logf(1.f + __expf(-fabsf(x))); }
__device__ __forceinline__ float prep_gate(int prep, float g) {
  return (prep & KDA_PREP_GATE_LOGSIGMOID) ? log_sigmoid(g) : g;
}
__device__ __forceinline__ float prep_beta(int prep, float b) { return (prep & KDA_PREP_BETA_SIGMOID) ? sigmoidf(b) : b; }

// Decay factor alpha = exp(g) of key channel c for one (token, head) whose
// per-channel gates start at g_chan and whose per-head gate is g_head
// (kda_gate: per channel, per head, or none); g prepared as `prep` says.
template <typename T>
__device__ __forceinline__ float gate_alpha(int gate, int prep, const T* g_chan, const T* g_head, int c) {
  if (gate == KDA_GATE_CHANNEL) return expf(prep_gate(prep, to_f32(g_chan[c])));
  if (gate == KDA_GATE_HEAD) return expf(prep_gate(prep, to_f32(*g_head)));
  return 1.f;
}

// Records events[i] on the stream when an events array was given.
inline cudaError_t mark(void* const* events, int i, cudaStream_t stream) {
  return events ? cudaEventRecord(static_cast<cudaEvent_t>(events[i]), stream) : cudaSuccess;
}

// Every workspace starts with this header; kernels that wait on barriers with
// an iteration limit record a give-up here instead of hanging.
struct WorkspaceHeader {
  unsigned int error;      // 0 = fine, nonzero = a bounded wait gave up
  unsigned int where;      // which wait (kernel-specific code)
  unsigned int pad[62];    // keeps the payload 256-byte aligned
};
static_assert(sizeof(WorkspaceHeader) == 256, "workspace header is 256 bytes");

}  // namespace kda
