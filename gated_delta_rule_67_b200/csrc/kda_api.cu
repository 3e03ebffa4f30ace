// kda_api.cu -- the C ABI of libkda.so: host-side validation and dispatch.
//
// Every argument is checked here, before anything is enqueued; the kernels
// themselves assume valid, aligned, non-overlapping buffers.
#include <string.h>

#include "kda_common.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_to(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct Range {
  const char* lo;
  size_t bytes;
};

bool overlaps(Range a, Range b) {
  if (!a.lo || !b.lo || a.bytes == 0 || b.bytes == 0) return false;
  return a.lo < b.lo + b.bytes && b.lo < a.lo + a.bytes;
}

size_t elem_bytes(int dtype) { return dtype == KDA_F32 ? 4 : 2; }

kda_status from_cuda(cudaError_t e) { return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA; }

bool prefill_supported(int dk, int dv, int chunk, int dtype) {
  if (dtype == KDA_F32)
    return (dk == 64 || dk == 128) && (dv == 64 || dv == 128) &&
           (chunk == 16 || chunk == 32 || chunk == 64);
  return (dk == 64 || dk == 128) && (dv == 64 || dv == 128) && chunk == 64;
}

}  // namespace

extern "C" {

const char* kda_status_string(int status) {
  switch (status) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG: null, misaligned, overlapping or out-of-range argument";
    case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED: valid arguments outside the implemented shapes/dtypes";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA: a CUDA runtime call or kernel launch failed";
    case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: a bounded on-device wait gave up";
    default: return "KDA_ERR_UNKNOWN: not a kda_status value";
  }
}

int kda_version(void) { return 100; }

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int chunk, int dtype) {
  if (B < 0 || T < 0 || H < 1 || dk < 1 || dv < 1 || chunk < 1) return 0;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return 0;
  if (!prefill_supported(dk, dv, chunk, dtype)) return 0;
  if (dtype == KDA_BF16) return kda::prefill_bf16_workspace_bytes(B, T, H, dk, dv, chunk);
  return 0;
}

int kda_chunk_fwd_launch_count(int B, int T, int H, int dk, int dv, int chunk, int dtype) {
  if (B < 0 || T < 0 || H < 1 || dk < 1 || dv < 1 || chunk < 1) return -1;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return -1;
  if (!prefill_supported(dk, dv, chunk, dtype)) return -1;
  if (B == 0 || T == 0) return 0;
  return dtype == KDA_BF16 ? kda::prefill_bf16_launches(B, T, H) : 1;
}

static kda_status chunk_fwd_impl(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                 float scale, const float* initial_state, void* o, float* final_state, int B,
                                 int T, int H, int dk, int dv, int chunk, int dtype, int gate, int prep,
                                 void* workspace, size_t workspace_bytes, void* stream_, void* const* events) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (B < 0 || T < 0 || H < 1 || dk < 1 || dv < 1 || chunk < 1) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (gate != KDA_GATE_CHANNEL && gate != KDA_GATE_HEAD && gate != KDA_GATE_NONE) return KDA_ERR_INVALID_ARG;
  if (prep & ~kda::kPrepMask) return KDA_ERR_INVALID_ARG;
  if (gate == KDA_GATE_NONE) g = nullptr;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return KDA_ERR_INVALID_ARG;
  const bool empty = (B == 0 || T == 0);
  const size_t eb = elem_bytes(dtype);
  const size_t ntok = (size_t)B * T * H;
  const Range rq{(const char*)q, ntok * dk * eb}, rk{(const char*)k, ntok * dk * eb},
      rg{(const char*)g, gate == KDA_GATE_CHANNEL ? ntok * dk * eb : ntok * eb}, rv{(const char*)v, ntok * dv * eb},
      rb{(const char*)beta, ntok * eb}, ro{(const char*)o, ntok * dv * eb};
  const size_t state_bytes = (size_t)B * H * dk * dv * sizeof(float);
  const Range rs0{(const char*)initial_state, state_bytes}, rsT{(const char*)final_state, state_bytes};
  if (!empty) {
    const void* need[] = {q, k, v, o};
    for (const void* p : need)
      if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARG;
    if (!beta || !aligned_to(beta, eb)) return KDA_ERR_INVALID_ARG;
    if (gate == KDA_GATE_CHANNEL && (!g || !aligned16(g))) return KDA_ERR_INVALID_ARG;
    if (gate == KDA_GATE_HEAD && (!g || !aligned_to(g, eb))) return KDA_ERR_INVALID_ARG;
    // o is written: it must not overlap any input.
    for (Range r : {rq, rk, rg, rv, rb, rs0})
      if (overlaps(ro, r)) return KDA_ERR_INVALID_ARG;
  }
  if (initial_state && !aligned16(initial_state)) return KDA_ERR_INVALID_ARG;
  if (final_state && !aligned16(final_state)) return KDA_ERR_INVALID_ARG;
  if (final_state && !empty) {
    for (Range r : {rq, rk, rg, rv, rb, ro})
      if (overlaps(rsT, r)) return KDA_ERR_INVALID_ARG;
    if (initial_state && (const void*)initial_state != (const void*)final_state && overlaps(rsT, rs0))
      return KDA_ERR_INVALID_ARG;
  }
  if (!prefill_supported(dk, dv, chunk, dtype)) return KDA_ERR_UNSUPPORTED;
  const size_t need_ws = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, chunk, dtype);
  if (need_ws > 0 && !empty) {
    if (!workspace || workspace_bytes < need_ws || (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return KDA_ERR_INVALID_ARG;
    const Range rw{(const char*)workspace, workspace_bytes};
    for (Range r : {rq, rk, rg, rv, rb, ro, rs0, rsT})
      if (overlaps(rw, r)) return KDA_ERR_INVALID_ARG;
  }

  if (events)
    for (int i = 0; i < 3; ++i)
      if (!events[i]) return KDA_ERR_INVALID_ARG;
  if (empty) {
    // Nothing to run: the final state is the initial state (or zeros).
    cudaError_t e = cudaSuccess;
    if (final_state && state_bytes && initial_state != final_state)
      e = initial_state ? cudaMemcpyAsync(final_state, initial_state, state_bytes, cudaMemcpyDeviceToDevice, stream)
                        : cudaMemsetAsync(final_state, 0, state_bytes, stream);
    for (int i = 0; i < 3 && e == cudaSuccess; ++i) e = kda::mark(events, i, stream);
    return from_cuda(e);
  }

  cudaError_t e;
  if (dtype == KDA_F32) {
    e = kda::launch_prefill_f32((const float*)q, (const float*)k, (const float*)v, (const float*)g,
                                (const float*)beta, scale, initial_state, (float*)o, final_state, B, T,
                                H, dk, dv, chunk, gate, prep, stream, events);
  } else {
    e = kda::launch_prefill_bf16((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                 (const __nv_bfloat16*)v, (const __nv_bfloat16*)g,
                                 (const __nv_bfloat16*)beta, scale, initial_state, (__nv_bfloat16*)o,
                                 final_state, B, T, H, dk, dv, chunk, gate, prep, workspace, workspace_bytes,
                                 stream, events);
  }
  return from_cuda(e);
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const void* g, const void* beta,
                         float scale, const float* initial_state, void* o, float* final_state, int B,
                         int T, int H, int dk, int dv, int chunk, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return chunk_fwd_impl(q, k, v, g, beta, scale, initial_state, o, final_state, B, T, H, dk, dv, chunk, dtype,
                        KDA_GATE_CHANNEL, KDA_PREP_NONE, workspace, workspace_bytes, stream, nullptr);
}

kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* g, const void* beta,
                            float scale, const float* initial_state, void* o, float* final_state, int B, int T,
                            int H, int dk, int dv, int chunk, int dtype, int gate, int prep, void* workspace,
                            size_t workspace_bytes, void* stream) {
  return chunk_fwd_impl(q, k, v, g, beta, scale, initial_state, o, final_state, B, T, H, dk, dv, chunk, dtype,
                        gate, prep, workspace, workspace_bytes, stream, nullptr);
}

kda_status kda_chunk_fwd_profiled(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                  float scale, const float* initial_state, void* o, float* final_state, int B,
                                  int T, int H, int dk, int dv, int chunk, int dtype, void* workspace,
                                  size_t workspace_bytes, void* stream, void* const* events) {
  if (!events) return KDA_ERR_INVALID_ARG;
  return chunk_fwd_impl(q, k, v, g, beta, scale, initial_state, o, final_state, B, T, H, dk, dv, chunk, dtype,
                        KDA_GATE_CHANNEL, KDA_PREP_NONE, workspace, workspace_bytes, stream, events);
}

kda_status kda_chunk_fwd_check(const void* workspace, size_t workspace_bytes, void* stream_) {
  if (!workspace || workspace_bytes < sizeof(kda::WorkspaceHeader)) return KDA_OK;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  kda::WorkspaceHeader h;
  cudaError_t e = cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return KDA_ERR_CUDA;
  return h.error ? KDA_ERR_TIMEOUT : KDA_OK;
}

kda_status kda_wait_selftest(void* workspace, size_t workspace_bytes, void* stream_) {
  if (!workspace || workspace_bytes < sizeof(kda::WorkspaceHeader) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return KDA_ERR_INVALID_ARG;
  return from_cuda(kda::launch_wait_selftest(workspace, static_cast<cudaStream_t>(stream_)));
}

size_t kda_backward_workspace_size(int B, int T, int H, int dk, int dv, int dtype) {
  if (B < 0 || T < 0 || H < 1) return 0;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return 0;
  if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return 0;
  return kda::backward_workspace_bytes(B, T, H, dk, dv, dtype);
}

size_t kda_backward_ex_workspace_size(int B, int T, int H, int dk, int dv, int dtype, int prep) {
  const size_t base = kda_backward_workspace_size(B, T, H, dk, dv, dtype);
  if (base == 0 || (prep & ~kda::kPrepMask)) return 0;
  return prep ? base + kda::backward_prep_bytes(B, T, H, dk, dtype) : base;
}

kda_status kda_backward(const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
                        const float* initial_state, const void* grad_o, const float* grad_final_state, void* grad_q,
                        void* grad_k, void* grad_v, void* grad_g, void* grad_beta, float* grad_initial_state, int B,
                        int T, int H, int dk, int dv, int dtype, int gate, void* workspace, size_t workspace_bytes,
                        void* stream_) {
  return kda_backward_ex(q, k, v, g, beta, scale, initial_state, grad_o, grad_final_state, grad_q, grad_k, grad_v,
                         grad_g, grad_beta, grad_initial_state, B, T, H, dk, dv, dtype, gate, KDA_PREP_NONE, workspace,
                         workspace_bytes, stream_);
}

kda_status kda_backward_ex(const void* q, const void* k, const void* v, const void* g, const void* beta, float scale,
                           const float* initial_state, const void* grad_o, const float* grad_final_state, void* grad_q,
                           void* grad_k, void* grad_v, void* grad_g, void* grad_beta, float* grad_initial_state, int B,
                           int T, int H, int dk, int dv, int dtype, int gate, int prep, void* workspace,
                           size_t workspace_bytes, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (B < 0 || T < 0 || H < 1 || dk < 1 || dv < 1) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (gate != KDA_GATE_CHANNEL && gate != KDA_GATE_HEAD && gate != KDA_GATE_NONE) return KDA_ERR_INVALID_ARG;
  if (prep & ~kda::kPrepMask) return KDA_ERR_INVALID_ARG;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return KDA_ERR_INVALID_ARG;
  if (gate == KDA_GATE_NONE) g = nullptr, grad_g = nullptr;
  const bool empty = (B == 0 || T == 0);
  const size_t eb = elem_bytes(dtype), ntok = (size_t)B * T * H, state_bytes = (size_t)B * H * dk * dv * 4;
  const size_t gbytes = gate == KDA_GATE_CHANNEL ? ntok * dk * eb : ntok * eb;
  const Range rq{(const char*)q, ntok * dk * eb}, rk{(const char*)k, ntok * dk * eb},
      rv{(const char*)v, ntok * dv * eb}, rg{(const char*)g, gbytes}, rb{(const char*)beta, ntok * eb},
      rs0{(const char*)initial_state, state_bytes}, rdo{(const char*)grad_o, ntok * dv * eb},
      rdsT{(const char*)grad_final_state, state_bytes};
  const Range wq{(const char*)grad_q, ntok * dk * eb}, wk{(const char*)grad_k, ntok * dk * eb},
      wv{(const char*)grad_v, ntok * dv * eb}, wg{(const char*)grad_g, gbytes}, wb{(const char*)grad_beta, ntok * eb},
      ws0{(const char*)grad_initial_state, state_bytes};
  if (!empty) {
    const void* need[] = {q, k, v, grad_o, grad_q, grad_k, grad_v};
    for (const void* p : need)
      if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARG;
    for (const void* p : {beta, (const void*)grad_beta})
      if (!p || !aligned_to(p, eb)) return KDA_ERR_INVALID_ARG;
    if (gate == KDA_GATE_CHANNEL && (!g || !grad_g || !aligned16(g) || !aligned16(grad_g))) return KDA_ERR_INVALID_ARG;
    if (gate == KDA_GATE_HEAD && (!g || !grad_g || !aligned_to(g, eb) || !aligned_to(grad_g, eb)))
      return KDA_ERR_INVALID_ARG;
  }
  for (const void* p : {(const void*)initial_state, (const void*)grad_final_state, (const void*)grad_initial_state})
    if (p && !aligned16(p)) return KDA_ERR_INVALID_ARG;
  const Range outs[] = {wq, wk, wv, wg, wb, ws0};
  for (int i = 0; i < 6; ++i) {
    for (Range r : {rq, rk, rv, rg, rb, rs0, rdo, rdsT})
      if (overlaps(outs[i], r)) return KDA_ERR_INVALID_ARG;
    for (int j = i + 1; j < 6; ++j)
      if (overlaps(outs[i], outs[j])) return KDA_ERR_INVALID_ARG;
  }
  if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
  if (empty) {  // dL/dS_0 = dL/dS_T
    cudaError_t e = cudaSuccess;
    if (grad_initial_state && state_bytes)
      e = grad_final_state ? cudaMemcpyAsync(grad_initial_state, grad_final_state, state_bytes,
                                             cudaMemcpyDeviceToDevice, stream)
                           : cudaMemsetAsync(grad_initial_state, 0, state_bytes, stream);
    return from_cuda(e);
  }
  // at least one (sequence, head)'s records, after the prepared inputs when `prep` is set
  const size_t prep_ws = prep ? kda::backward_prep_bytes(B, T, H, dk, dtype) : 0;
  const size_t need_ws = prep_ws + kda::backward_workspace_bytes(1, T, 1, dk, dv, dtype);
  if (!workspace || workspace_bytes < need_ws || !aligned16(workspace)) return KDA_ERR_INVALID_ARG;
  const Range rw{(const char*)workspace, workspace_bytes};
  for (Range r : {rq, rk, rv, rg, rb, rs0, rdo, rdsT, wq, wk, wv, wg, wb, ws0})
    if (overlaps(rw, r)) return KDA_ERR_INVALID_ARG;
  if (prep)
    return from_cuda(kda::launch_backward_prepared(q, k, v, g, beta, scale, initial_state, grad_o, grad_final_state,
                                                   grad_q, grad_k, grad_v, grad_g, grad_beta, grad_initial_state, B,
                                                   T, H, dk, dv, dtype, gate, prep, workspace, workspace_bytes,
                                                   stream));
  return from_cuda(kda::launch_backward(q, k, v, g, beta, scale, initial_state, grad_o, grad_final_state, grad_q,
                                        grad_k, grad_v, grad_g, grad_beta, grad_initial_state, B, T, H, dk, dv, dtype,
                                        gate, workspace, workspace_bytes, stream));
}

static kda_status recurrent_step_impl(const void* q, const void* k, const void* v, const void* g,
                                      const void* beta, float scale, float* state, void* o, int N, int H, int dk,
                                      int dv, int dtype, int gate, int prep, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (N < 0 || H < 1 || dk < 1 || dv < 1) return KDA_ERR_INVALID_ARG;
  if (dtype != KDA_F32 && dtype != KDA_BF16) return KDA_ERR_INVALID_ARG;
  if (gate != KDA_GATE_CHANNEL && gate != KDA_GATE_HEAD && gate != KDA_GATE_NONE) return KDA_ERR_INVALID_ARG;
  if (prep & ~kda::kPrepMask) return KDA_ERR_INVALID_ARG;
  if (gate == KDA_GATE_NONE) g = nullptr;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return KDA_ERR_INVALID_ARG;
  if (N == 0) return KDA_OK;
  const size_t eb = elem_bytes(dtype);
  const void* need[] = {q, k, v, state, o};
  for (const void* p : need)
    if (!p || !aligned16(p)) return KDA_ERR_INVALID_ARG;
  if (!beta || !aligned_to(beta, eb)) return KDA_ERR_INVALID_ARG;
  if (gate == KDA_GATE_CHANNEL && (!g || !aligned16(g))) return KDA_ERR_INVALID_ARG;
  if (gate == KDA_GATE_HEAD && (!g || !aligned_to(g, eb))) return KDA_ERR_INVALID_ARG;
  const size_t nh = (size_t)N * H;
  const Range rq{(const char*)q, nh * dk * eb}, rk{(const char*)k, nh * dk * eb},
      rg{(const char*)g, gate == KDA_GATE_CHANNEL ? nh * dk * eb : nh * eb}, rv{(const char*)v, nh * dv * eb},
      rb{(const char*)beta, nh * eb}, ro{(const char*)o, nh * dv * eb},
      rs{(const char*)state, nh * dk * dv * sizeof(float)};
  for (Range r : {rq, rk, rg, rv, rb, rs})
    if (overlaps(ro, r)) return KDA_ERR_INVALID_ARG;
  for (Range r : {rq, rk, rg, rv, rb})
    if (overlaps(rs, r)) return KDA_ERR_INVALID_ARG;
  if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_UNSUPPORTED;
  return from_cuda(kda::launch_decode(q, k, v, g, beta, scale, state, o, N, H, dk, dv, dtype, gate, prep, stream));
}

kda_status kda_recurrent_step(const void* q, const void* k, const void* v, const void* g,
                              const void* beta, float scale, float* state, void* o, int N, int H,
                              int dk, int dv, int dtype, void* stream) {
  return recurrent_step_impl(q, k, v, g, beta, scale, state, o, N, H, dk, dv, dtype, KDA_GATE_CHANNEL,
                             KDA_PREP_NONE, stream);
}

kda_status kda_recurrent_step_ex(const void* q, const void* k, const void* v, const void* g,
                                 const void* beta, float scale, float* state, void* o, int N, int H,
                                 int dk, int dv, int dtype, int gate, int prep, void* stream) {
  return recurrent_step_impl(q, k, v, g, beta, scale, state, o, N, H, dk, dv, dtype, gate, prep, stream);
}

}  // extern "C"
