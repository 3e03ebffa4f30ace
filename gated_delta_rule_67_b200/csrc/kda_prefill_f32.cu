// kda_prefill_f32.cu -- fp32 KDA prefill on CUDA cores (FFMA).
//
// For fp32 inputs the library keeps full fp32 arithmetic: the tf32 tensor-core
// formats carry a 10-bit mantissa, too coarse for a 1e-4 relative bound, so
// this path runs the KDA recurrence (KimiLinear article, section 2.3) token
// by token on the CUDA cores.  The columns of the state evolve independently
// (column j only ever meets column j of v and of o), so the state is split by
// columns across CTAs and threads:
//     CTA   = (b, h, 32 value columns)
//     thread = (column, row group rg in 0..3); it owns rows rg, rg+4, ...
// The per-token reductions over the key channels (S'^T k and S^T q) are
// 4-lane butterflies.  Tokens are staged through shared memory in tiles of
// kTile; the caller's chunk size does not change the arithmetic.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kCols = 32;   // value columns per CTA
constexpr int kGroups = 4;  // row groups per column
constexpr int kTile = 16;   // tokens staged per shared-memory tile

template <int DK>
__global__ void __launch_bounds__(kCols * kGroups)
    prefill_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                       const float* __restrict__ v, const float* __restrict__ g,
                       const float* __restrict__ beta, float scale, const float* __restrict__ s0,
                       float* __restrict__ o, float* sT, int T, int H, int DV, int gate, int prep) {
  constexpr int RW = DK / kGroups;
  __shared__ float sq[kTile][DK], sk[kTile][DK], sa[kTile][DK];
  __shared__ float sv[kTile][kCols], sb[kTile];

  const int tid = threadIdx.x;
  const int rg = tid & (kGroups - 1);
  const int cl = tid / kGroups;
  const int col = blockIdx.x * kCols + cl;
  const int h = blockIdx.y, b = blockIdx.z;
  const size_t state_off = ((size_t)b * H + h) * DK * DV;

  float s[RW];
#pragma unroll
  for (int i = 0; i < RW; ++i) s[i] = s0 ? s0[state_off + (size_t)(i * kGroups + rg) * DV + col] : 0.f;

  for (int t0 = 0; t0 < T; t0 += kTile) {
    const int nt = min(kTile, T - t0);
    __syncthreads();
    for (int e = tid; e < nt * DK; e += blockDim.x) {
      const int tt = e / DK, c = e % DK;
      const size_t tok = ((size_t)b * T + t0 + tt) * H + h, off = tok * DK + c;
      sq[tt][c] = q[off];
      sk[tt][c] = k[off];
      sa[tt][c] = gate_alpha(gate, prep, g + tok * DK, g + tok, c);
    }
    for (int e = tid; e < nt * kCols; e += blockDim.x) {
      const int tt = e / kCols, c = e % kCols;
      sv[tt][c] = v[(((size_t)b * T + t0 + tt) * H + h) * DV + blockIdx.x * kCols + c];
    }
    if (tid < nt) sb[tid] = prep_beta(prep, beta[((size_t)b * T + t0 + tid) * H + h]);
    __syncthreads();
    if (prep & KDA_PREP_L2NORM_QK) {  // q, k of each staged token to unit length: 8 threads per token
      static_assert(kCols * kGroups == 8 * kTile, "8 threads per staged token");
      const int tt = tid >> 3, part = tid & 7;
      constexpr int PW = DK / 8;
      float qs = 0.f, ks = 0.f;
#pragma unroll
      for (int c = 0; c < PW; ++c) {
        qs = fmaf(sq[tt][part * PW + c], sq[tt][part * PW + c], qs);
        ks = fmaf(sk[tt][part * PW + c], sk[tt][part * PW + c], ks);
      }
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) {
        qs += __shfl_xor_sync(0xffffffffu, qs, off);
        ks += __shfl_xor_sync(0xffffffffu, ks, off);
      }
      const float rq = rsqrtf(qs + kL2Eps), rk = rsqrtf(ks + kL2Eps);
#pragma unroll
      for (int c = 0; c < PW; ++c) {
        sq[tt][part * PW + c] *= rq;
        sk[tt][part * PW + c] *= rk;
      }
      __syncthreads();
    }

    for (int tt = 0; tt < nt; ++tt) {
      float pk = 0.f;
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int row = i * kGroups + rg;
        s[i] *= sa[tt][row];
        pk = fmaf(sk[tt][row], s[i], pk);
      }
      pk += __shfl_xor_sync(0xffffffffu, pk, 1);
      pk += __shfl_xor_sync(0xffffffffu, pk, 2);
      const float u = sb[tt] * (sv[tt][cl] - pk);
      float pq = 0.f;
#pragma unroll
      for (int i = 0; i < RW; ++i) {
        const int row = i * kGroups + rg;
        s[i] = fmaf(sk[tt][row], u, s[i]);
        pq = fmaf(sq[tt][row], s[i], pq);
      }
      pq += __shfl_xor_sync(0xffffffffu, pq, 1);
      pq += __shfl_xor_sync(0xffffffffu, pq, 2);
      if (rg == 0) o[(((size_t)b * T + t0 + tt) * H + h) * DV + col] = scale * pq;
    }
  }
  if (sT) {
#pragma unroll
    for (int i = 0; i < RW; ++i) sT[state_off + (size_t)(i * kGroups + rg) * DV + col] = s[i];
  }
}

}  // namespace

cudaError_t launch_prefill_f32(const float* q, const float* k, const float* v, const float* g,
                               const float* beta, float scale, const float* s0, float* o, float* sT,
                               int B, int T, int H, int dk, int dv, int chunk, int gate, int prep,
                               cudaStream_t stream, void* const* events) {
  (void)chunk;
  dim3 grid(dv / kCols, H, B);
  cudaError_t e = mark(events, 0, stream);
  if (e != cudaSuccess) return e;
  if (dk == 128)
    prefill_f32_kernel<128><<<grid, kCols * kGroups, 0, stream>>>(q, k, v, g, beta, scale, s0, o, sT, T, H, dv, gate, prep);
  else
    prefill_f32_kernel<64><<<grid, kCols * kGroups, 0, stream>>>(q, k, v, g, beta, scale, s0, o, sT, T, H, dv, gate, prep);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = mark(events, 1, stream);
  if (e == cudaSuccess) e = mark(events, 2, stream);
  return e;
}

}  // namespace kda
