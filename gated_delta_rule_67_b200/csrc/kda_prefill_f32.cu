// kda_prefill_f32.cu -- fp32 chunked KDA prefill on CUDA cores (FFMA).
//
// For fp32 inputs the library keeps full fp32 arithmetic: the tf32 tensor-core
// formats carry a 10-bit mantissa, too coarse for a 1e-4 relative bound.  The
// chunkwise algorithm of the KimiLinear article (section 3.1; the update is
// section 2.3) runs here with the caller's chunk size C in {16, 32, 64}: per
// chunk, with G the in-chunk cumulative log-gate and S0 the entering state,
//
//   A_kk[i,j] = beta_i sum_c k_ic k_jc exp(G_ic - G_jc)      (j < i)
//   A_qk[i,j] = scale sum_c q_ic k_jc exp(G_ic - G_jc)       (j <= i)
//   (I + A_kk) [W | U] = diag(beta) [K+ | V]                  (forward substitution)
//   V' = U - W S0,   O = Q+ S0 + A_qk V',   S = Diag(exp(G_C)) S0 + Kbar^T V'
//
// with K+ = k exp(G), Q+ = scale q exp(G), Kbar = k exp(G_C - G).  Every
// decay factor is formed as exp of a difference that is <= 0 for gates in
// (0, 1] (the pairwise factors of the score matrices per (pair, channel)), so
// no factor can overflow whatever the gates; the chunk size changes the
// arithmetic (C(C+1)/2 pairs per chunk, C sequential substitution steps) but
// not the result.  The columns of the state evolve independently, so a CTA
// owns one (sequence, head) and 32 value columns; the chunk's score matrices
// and W are recomputed by every column slice of the same head.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kCols = 32;      // value columns per CTA
constexpr int kThreads = 256;

// Shared-memory plan (floats): rows of the [C][DK] tiles are padded to DK + 1
// so that threads reading different rows at one channel hit different banks.
template <int DK, int C>
struct F32Plan {
  static constexpr int P = DK + 1;
  static constexpr int k = 0;                    // [C][P] k
  static constexpr int G = k + C * P;            // [C][P] cumulative log-gate
  static constexpr int Q = G + C * P;            // [C][P] q -> Q+
  static constexpr int W = Q + C * P;            // [C][P] K+ -> W -> Kbar
  static constexpr int A = W + C * P;            // [C][C] A_kk (strictly lower, times beta_i)
  static constexpr int Aq = A + C * C;           // [C][C] A_qk (lower)
  static constexpr int U = Aq + C * C;           // [C][kCols] v -> U
  static constexpr int V = U + C * kCols;        // [C][kCols] V'
  static constexpr int S = V + C * kCols;        // [DK][kCols] state slice
  static constexpr int b = S + DK * kCols;       // [C] beta
  static constexpr int nq = b + C;               // [C] unit-length factor of q (fused preparation)
  static constexpr int nk = nq + C;              // [C] unit-length factor of k
  static constexpr int floats = nk + C;
  static constexpr size_t bytes = (size_t)floats * sizeof(float);
};

template <int DK, int C>
__global__ void __launch_bounds__(kThreads)
    prefill_f32_chunk_kernel(const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
                             const float* __restrict__ g, const float* __restrict__ beta, float scale,
                             const float* __restrict__ s0, float* __restrict__ o, float* sT, int T, int H, int DV,
                             int gate, int prep) {
  using Pl = F32Plan<DK, C>;
  constexpr int P = Pl::P;
  extern __shared__ float smf[];
  float *sk = smf + Pl::k, *sG = smf + Pl::G, *sQ = smf + Pl::Q, *sW = smf + Pl::W;
  float *sA = smf + Pl::A, *sAq = smf + Pl::Aq, *sU = smf + Pl::U, *sV = smf + Pl::V, *sS = smf + Pl::S;
  float *sb = smf + Pl::b, *snq = smf + Pl::nq, *snk = smf + Pl::nk;

  const int tid = threadIdx.x;
  const int cs = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t state_off = ((size_t)b * H + h) * DK * DV + (size_t)cs * kCols;
  const bool l2n = prep & KDA_PREP_L2NORM_QK;

  for (int e = tid; e < DK * kCols; e += kThreads) {
    const int c = e / kCols, col = e % kCols;
    sS[c * kCols + col] = s0 ? s0[state_off + (size_t)c * DV + col] : 0.f;
  }

  for (int t0 = 0; t0 < T; t0 += C) {
    const int L = min(C, T - t0);
    __syncthreads();  // the previous chunk is done with every tile
    // ---- the chunk's inputs (zero past the end: zero k, q, v, beta and gate add nothing)
    for (int e = tid; e < C * DK; e += kThreads) {
      const int t = e / DK, c = e % DK;
      const bool valid = t < L;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      float gv = 0.f;
      if (valid && gate == KDA_GATE_CHANNEL) gv = prep_gate(prep, g[tok * DK + c]);
      if (valid && gate == KDA_GATE_HEAD) gv = prep_gate(prep, g[tok]);
      sk[t * P + c] = valid ? k[tok * DK + c] : 0.f;
      sQ[t * P + c] = valid ? q[tok * DK + c] : 0.f;
      sG[t * P + c] = gv;
    }
    for (int e = tid; e < C * kCols; e += kThreads) {
      const int t = e / kCols, col = e % kCols;
      sU[e] = t < L ? v[(((size_t)b * T + t0 + t) * H + h) * DV + cs * kCols + col] : 0.f;
    }
    if (tid < C) sb[tid] = tid < L ? prep_beta(prep, beta[((size_t)b * T + t0 + tid) * H + h]) : 0.f;
    __syncthreads();
    if (l2n) {  // q and k of each token to unit length: 256 / C threads per token
      constexpr int per = kThreads / C;
      const int t = tid / per, part = tid % per;
      float qs = 0.f, ks = 0.f;
      for (int c = part; c < DK; c += per) {
        qs = fmaf(sQ[t * P + c], sQ[t * P + c], qs);
        ks = fmaf(sk[t * P + c], sk[t * P + c], ks);
      }
#pragma unroll
      for (int off = per / 2; off > 0; off >>= 1) {
        qs += __shfl_xor_sync(0xffffffffu, qs, off);
        ks += __shfl_xor_sync(0xffffffffu, ks, off);
      }
      if (part == 0) {
        snq[t] = rsqrtf(qs + kL2Eps);
        snk[t] = rsqrtf(ks + kL2Eps);
      }
      __syncthreads();
      for (int e = tid; e < C * DK; e += kThreads) {
        const int t2 = e / DK, c = e % DK;
        sQ[t2 * P + c] *= snq[t2];
        sk[t2 * P + c] *= snk[t2];
      }
    }
    // ---- cumulative log-gate, one channel per thread
    if (tid < DK) {
      float a = 0.f;
#pragma unroll 4
      for (int t = 0; t < C; ++t) {
        a += sG[t * P + tid];
        sG[t * P + tid] = a;
      }
    }
    __syncthreads();
    // ---- score matrices, pair by pair, every decay factor exp(G_i - G_j) formed per channel
    constexpr int kPairs = C * (C + 1) / 2;
    for (int p = tid; p < kPairs; p += kThreads) {
      int i = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
      while (i * (i + 1) / 2 > p) --i;
      while ((i + 1) * (i + 2) / 2 <= p) ++i;
      const int j = p - i * (i + 1) / 2;
      float akk = 0.f, aqk = 0.f;
#pragma unroll 4
      for (int c = 0; c < DK; ++c) {
        const float d = expf(sG[i * P + c] - sG[j * P + c]);
        const float kj = sk[j * P + c] * d;
        akk = fmaf(sk[i * P + c], kj, akk);
        aqk = fmaf(sQ[i * P + c], kj, aqk);
      }
      sA[i * C + j] = j < i ? sb[i] * akk : 0.f;
      sAq[i * C + j] = scale * aqk;
    }
    for (int e = tid; e < C * C; e += kThreads) {
      const int i = e / C, j = e % C;
      if (j > i) sA[e] = sAq[e] = 0.f;
      if (j == i) sA[e] = 0.f;
    }
    __syncthreads();
    // ---- start-decayed operands K+ = k exp(G), Q+ = scale q exp(G) (factors <= 1)
    for (int e = tid; e < C * DK; e += kThreads) {
      const int t = e / DK, c = e % DK;
      const float eg = expf(sG[t * P + c]);
      sW[t * P + c] = sk[t * P + c] * eg;
      sQ[t * P + c] = scale * sQ[t * P + c] * eg;
    }
    __syncthreads();
    // ---- (I + A_kk) [W | U] = diag(beta) [K+ | V]: one column per thread, rows in order
    for (int col = tid; col < DK + kCols; col += kThreads) {
      float* X = col < DK ? sW + col : sU + (col - DK);
      const int stride = col < DK ? P : kCols;
      for (int i = 0; i < C; ++i) {
        float x = sb[i] * X[i * stride];
        for (int m = 0; m < i; ++m) x = fmaf(-sA[i * C + m], X[m * stride], x);
        X[i * stride] = x;
      }
    }
    __syncthreads();
    // ---- V' = U - W S0
    for (int e = tid; e < C * kCols; e += kThreads) {
      const int i = e / kCols, col = e % kCols;
      float x = sU[e];
#pragma unroll 8
      for (int c = 0; c < DK; ++c) x = fmaf(-sW[i * P + c], sS[c * kCols + col], x);
      sV[e] = x;
    }
    __syncthreads();
    // ---- O = Q+ S0 + A_qk V' for the chunk's tokens
    for (int e = tid; e < C * kCols; e += kThreads) {
      const int i = e / kCols, col = e % kCols;
      if (i >= L) continue;
      float x = 0.f;
#pragma unroll 8
      for (int c = 0; c < DK; ++c) x = fmaf(sQ[i * P + c], sS[c * kCols + col], x);
      for (int m = 0; m <= i; ++m) x = fmaf(sAq[i * C + m], sV[m * kCols + col], x);
      o[(((size_t)b * T + t0 + i) * H + h) * DV + cs * kCols + col] = x;
    }
    // ---- end-decayed keys Kbar = k exp(G_C - G) over W (read by now)
    __syncthreads();
    for (int e = tid; e < C * DK; e += kThreads) {
      const int t = e / DK, c = e % DK;
      sW[t * P + c] = sk[t * P + c] * expf(sG[(C - 1) * P + c] - sG[t * P + c]);
    }
    __syncthreads();
    // ---- S = Diag(exp(G_C)) S0 + Kbar^T V'
    for (int e = tid; e < DK * kCols; e += kThreads) {
      const int c = e / kCols, col = e % kCols;
      float x = expf(sG[(C - 1) * P + c]) * sS[e];
#pragma unroll 8
      for (int m = 0; m < C; ++m) x = fmaf(sW[m * P + c], sV[m * kCols + col], x);
      sS[e] = x;
    }
  }
  __syncthreads();
  if (sT) {
    for (int e = tid; e < DK * kCols; e += kThreads) {
      const int c = e / kCols, col = e % kCols;
      sT[state_off + (size_t)c * DV + col] = sS[e];
    }
  }
}

template <int DK, int C>
cudaError_t launch_f32(dim3 grid, cudaStream_t stream, const float* q, const float* k, const float* v, const float* g,
                       const float* beta, float scale, const float* s0, float* o, float* sT, int T, int H, int dv,
                       int gate, int prep) {
  // Function attributes belong to each device's context: set them once per
  // device (one bit per device ordinal; ordinals past 63 set them every call).
  static unsigned long long done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
  if (!(__atomic_load_n(&done, __ATOMIC_ACQUIRE) & bit) || !bit) {
    e = cudaFuncSetAttribute(prefill_f32_chunk_kernel<DK, C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)F32Plan<DK, C>::bytes);
    if (e != cudaSuccess) return e;
    __atomic_fetch_or(&done, bit, __ATOMIC_RELEASE);
  }
  prefill_f32_chunk_kernel<DK, C><<<grid, kThreads, F32Plan<DK, C>::bytes, stream>>>(q, k, v, g, beta, scale, s0, o,
                                                                                      sT, T, H, dv, gate, prep);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_f32(const float* q, const float* k, const float* v, const float* g,
                               const float* beta, float scale, const float* s0, float* o, float* sT,
                               int B, int T, int H, int dk, int dv, int chunk, int gate, int prep,
                               cudaStream_t stream, void* const* events) {
  dim3 grid(dv / kCols, H, B);
  cudaError_t e = mark(events, 0, stream);
  if (e != cudaSuccess) return e;
#define KDA_F32_CASE(DK, C)                                                                                   \
  if (dk == DK && chunk == C)                                                                                 \
    e = launch_f32<DK, C>(grid, stream, q, k, v, g, beta, scale, s0, o, sT, T, H, dv, gate, prep);
  KDA_F32_CASE(64, 16)
  KDA_F32_CASE(64, 32)
  KDA_F32_CASE(64, 64)
  KDA_F32_CASE(128, 16)
  KDA_F32_CASE(128, 32)
  KDA_F32_CASE(128, 64)
#undef KDA_F32_CASE
  if (e == cudaSuccess) e = mark(events, 1, stream);
  if (e == cudaSuccess) e = mark(events, 2, stream);
  return e;
}

}  // namespace kda
