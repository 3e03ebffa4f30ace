// kda_backward_prep.cu -- the backward pass through the fused input preparation.
//
// The forward (kda_chunk_fwd_ex with kda_prep bits) prepares raw inputs in its
// kernels: q, k scaled to unit length per token and head (r = (sum q^2 +
// 1e-6)^-1/2), g <- log sigmoid(g), beta <- sigmoid(beta).  The backward with
// the same bits runs in three steps:
//   1. bwd_prepare_kernel: the prepared q, k, g, beta into the workspace
//      (input dtype) and the per-row factors r of q and k (fp32);
//   2. the chunkwise backward on the prepared inputs, its gradients written
//      to the caller's gradient buffers (dq^ and dk^ to fp32 workspace
//      buffers for bf16 inputs: the L2 step's chain rule subtracts their
//      radial part, which bf16 rounding would not survive);
//   3. bwd_chain_kernel, in place on those buffers: the chain rule of each
//      step, dq = r (dq^ - q^ (q^ . dq^)) (same for k), dg = dg^ sigmoid(-g),
//      dbeta = dbeta^ sigmoid(beta) (1 - sigmoid(beta)), in fp32.
// One warp per (token, head) row in both kernels; sums over the key channels
// are warp reductions in a fixed order.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kRowsPerBlock = 8;  // warps per block, one (token, head) row each

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

struct PrepArgs {
  const void *q, *k, *g, *beta;   // raw inputs
  void *qh, *kh, *gh, *bh;        // prepared copies (workspace)
  float *rq, *rk;                 // per-row factors (workspace)
  float *dq32, *dk32;             // bf16 inputs: dq^, dk^ in fp32 (workspace); null for fp32 inputs
  void *dq, *dk, *dg, *dbeta;     // gradients, prepared space on entry to step 3, raw space after
  size_t rows;                    // B * T * H
  int prep, gate;
};

template <typename IO, int DK>
__global__ void __launch_bounds__(32 * kRowsPerBlock) bwd_prepare_kernel(const PrepArgs a) {
  constexpr int E = DK / 32;  // channels per lane
  const size_t row = (size_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  if (row >= a.rows) return;
  const int lane = threadIdx.x & 31;
  const bool l2 = a.prep & KDA_PREP_L2NORM_QK;
  for (int which = 0; which < 2; ++which) {
    const IO* x = static_cast<const IO*>(which ? a.k : a.q) + row * DK;
    IO* xh = static_cast<IO*>(which ? a.kh : a.qh) + row * DK;
    float v[E], ss = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      v[e] = to_f32(x[lane + 32 * e]);
      ss = fmaf(v[e], v[e], ss);
    }
    const float r = l2 ? rsqrtf(warp_sum(ss) + kL2Eps) : 1.f;
#pragma unroll
    for (int e = 0; e < E; ++e) xh[lane + 32 * e] = from_f32<IO>(v[e] * r);
    if (lane == 0) (which ? a.rk : a.rq)[row] = r;
  }
  if (a.gate == KDA_GATE_CHANNEL) {
    const IO* g = static_cast<const IO*>(a.g) + row * DK;
    IO* gh = static_cast<IO*>(a.gh) + row * DK;
#pragma unroll
    for (int e = 0; e < E; ++e) gh[lane + 32 * e] = from_f32<IO>(prep_gate(a.prep, to_f32(g[lane + 32 * e])));
  } else if (a.gate == KDA_GATE_HEAD && lane == 0) {
    static_cast<IO*>(a.gh)[row] = from_f32<IO>(prep_gate(a.prep, to_f32(static_cast<const IO*>(a.g)[row])));
  }
  if (lane == 0)
    static_cast<IO*>(a.bh)[row] = from_f32<IO>(prep_beta(a.prep, to_f32(static_cast<const IO*>(a.beta)[row])));
}

template <typename IO, int DK>
__global__ void __launch_bounds__(32 * kRowsPerBlock) bwd_chain_kernel(const PrepArgs a) {
  constexpr int E = DK / 32;
  const size_t row = (size_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 5);
  if (row >= a.rows) return;
  const int lane = threadIdx.x & 31;
  if (a.prep & KDA_PREP_L2NORM_QK) {
    for (int which = 0; which < 2; ++which) {
      const IO* xh = static_cast<const IO*>(which ? a.kh : a.qh) + row * DK;
      IO* d = static_cast<IO*>(which ? a.dk : a.dq) + row * DK;
      const float* d32 = which ? a.dk32 : a.dq32;  // dq^ (dk^) in fp32 when the outputs are bf16
      const float r = (which ? a.rk : a.rq)[row];
      float h[E], dh[E], dot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        h[e] = to_f32(xh[lane + 32 * e]);
        dh[e] = d32 ? d32[row * DK + lane + 32 * e] : to_f32(d[lane + 32 * e]);
        dot = fmaf(h[e], dh[e], dot);
      }
      dot = warp_sum(dot);
#pragma unroll
      for (int e = 0; e < E; ++e) d[lane + 32 * e] = from_f32<IO>(r * fmaf(-h[e], dot, dh[e]));
    }
  }
  if ((a.prep & KDA_PREP_GATE_LOGSIGMOID) && a.gate != KDA_GATE_NONE) {
    const int n = a.gate == KDA_GATE_CHANNEL ? DK : 1;
    const IO* g = static_cast<const IO*>(a.g) + row * n;
    IO* d = static_cast<IO*>(a.dg) + row * n;
    for (int c = lane; c < n; c += 32) d[c] = from_f32<IO>(to_f32(d[c]) * sigmoidf(-to_f32(g[c])));
  }
  if ((a.prep & KDA_PREP_BETA_SIGMOID) && lane == 0) {
    const float s = sigmoidf(to_f32(static_cast<const IO*>(a.beta)[row]));
    IO* d = static_cast<IO*>(a.dbeta) + row;
    *d = from_f32<IO>(to_f32(*d) * s * (1.f - s));
  }
}

template <typename IO>
cudaError_t launch_pair(bool chain, const PrepArgs& a, int dk, cudaStream_t stream) {
  const unsigned blocks = (unsigned)((a.rows + kRowsPerBlock - 1) / kRowsPerBlock);
  if (dk == 128) {
    if (chain)
      bwd_chain_kernel<IO, 128><<<blocks, 32 * kRowsPerBlock, 0, stream>>>(a);
    else
      bwd_prepare_kernel<IO, 128><<<blocks, 32 * kRowsPerBlock, 0, stream>>>(a);
  } else {
    if (chain)
      bwd_chain_kernel<IO, 64><<<blocks, 32 * kRowsPerBlock, 0, stream>>>(a);
    else
      bwd_prepare_kernel<IO, 64><<<blocks, 32 * kRowsPerBlock, 0, stream>>>(a);
  }
  return cudaGetLastError();
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t backward_prep_bytes(int B, int T, int H, int dk, int dtype) {
  const size_t rows = (size_t)B * T * H, eb = dtype == KDA_F32 ? 4 : 2;
  const size_t grads32 = dtype == KDA_F32 ? 0 : 2 * align256(rows * dk * 4);
  return 3 * align256(rows * dk * eb) + align256(rows * eb) + 2 * align256(rows * 4) + grads32;
}

cudaError_t launch_backward_prepared(const void* q, const void* k, const void* v, const void* g, const void* beta,
                                     float scale, const float* s0, const void* d_o, const float* dsT, void* dq,
                                     void* dk_out, void* dv_out, void* dg, void* dbeta, float* ds0, int B, int T, int H,
                                     int dk, int dv, int dtype, int gate, int prep, void* ws, size_t ws_bytes,
                                     cudaStream_t stream) {
  const size_t rows = (size_t)B * T * H, eb = dtype == KDA_F32 ? 4 : 2;
  // the error word of the backward's bounded waits leads the workspace, then the prepared inputs
  WorkspaceHeader* hdr = static_cast<WorkspaceHeader*>(ws);
  uint8_t* w = static_cast<uint8_t*>(ws) + sizeof(WorkspaceHeader);
  PrepArgs a;
  a.q = q, a.k = k, a.g = g, a.beta = beta;
  a.qh = w, w += align256(rows * dk * eb);
  a.kh = w, w += align256(rows * dk * eb);
  a.gh = w, w += align256(rows * dk * eb);
  a.bh = w, w += align256(rows * eb);
  a.rq = reinterpret_cast<float*>(w), w += align256(rows * 4);
  a.rk = reinterpret_cast<float*>(w), w += align256(rows * 4);
  a.dq32 = a.dk32 = nullptr;
  if (dtype != KDA_F32 && (prep & KDA_PREP_L2NORM_QK)) {  // only the L2 step's chain rule reads them
    a.dq32 = reinterpret_cast<float*>(w), w += align256(rows * dk * 4);
    a.dk32 = reinterpret_cast<float*>(w), w += align256(rows * dk * 4);
  }
  a.dq = dq, a.dk = dk_out, a.dg = dg, a.dbeta = dbeta;
  a.rows = rows, a.prep = prep, a.gate = gate;
  const size_t used = static_cast<size_t>(w - static_cast<uint8_t*>(ws));
  cudaError_t e = dtype == KDA_F32 ? launch_pair<float>(false, a, dk, stream)
                                   : launch_pair<__nv_bfloat16>(false, a, dk, stream);
  if (e != cudaSuccess) return e;
  e = launch_backward(a.qh, a.kh, v, gate == KDA_GATE_NONE ? nullptr : a.gh, a.bh, scale, s0, d_o, dsT, dq, dk_out,
                      dv_out, dg, dbeta, ds0, B, T, H, dk, dv, dtype, gate, w, ws_bytes - used, stream, a.dq32, a.dk32,
                      hdr);
  if (e != cudaSuccess) return e;
  return dtype == KDA_F32 ? launch_pair<float>(true, a, dk, stream) : launch_pair<__nv_bfloat16>(true, a, dk, stream);
}

}  // namespace kda
