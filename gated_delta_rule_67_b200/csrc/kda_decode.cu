// kda_decode.cu -- single-token KDA decode step (HBM-bound state stream).
//
// One step of the KDA recurrence (KimiLinear article, section 2.3; O(1)
// per-token decoding with a fixed-size state, section 4.2) for every
// (sequence, head):
//     S' = Diag(exp g) S                 decay the key-channel rows
//     u  = beta (v - S'^T k)             delta-rule correction
//     S  = S' + k u^T                    rank-1 write, stored in place
//     o  = scale S^T q = scale (S'^T q + (k.q) u)
//
// Cost model: each head's fp32 state (dk*dv*4 bytes, 64 KiB at d=128) is read
// once and written once; everything else is < 1% of the bytes.  One CTA per
// head, 8 warps; warp w owns dk/8 consecutive rows and lane l owns dv/32
// consecutive columns, so every state row is one coalesced 128-bit-per-lane
// warp access.  All of a thread's state loads are issued before any use
// (64 KiB in flight per CTA).  The two column reductions over dk (S'^T k and
// S'^T q) are split across warps and combined through shared memory.
#include "kda_common.cuh"

namespace kda {
namespace {

template <int CL>
struct Vec;
template <>
struct Vec<4> {
  __device__ static void load(const float* p, float* r) {
    float4 x = __ldcs(reinterpret_cast<const float4*>(p));
    r[0] = x.x; r[1] = x.y; r[2] = x.z; r[3] = x.w;
  }
  __device__ static void store(float* p, const float* r) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(r[0], r[1], r[2], r[3]));
  }
};
template <>
struct Vec<2> {
  __device__ static void load(const float* p, float* r) {
    float2 x = __ldcs(reinterpret_cast<const float2*>(p));
    r[0] = x.x; r[1] = x.y;
  }
  __device__ static void store(float* p, const float* r) {
    __stcs(reinterpret_cast<float2*>(p), make_float2(r[0], r[1]));
  }
};

constexpr int kDecodeWarps = 8;

// kGeneric: a forget gate other than per channel, or fused input preparation
// (run-time `gate` and `prep`); the default instance is the plain KDA step.
template <typename T, int DK, int DV, bool kGeneric>
__global__ void __launch_bounds__(kDecodeWarps * 32)
    decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       const T* __restrict__ g, const T* __restrict__ beta, float scale,
                       float* __restrict__ state, T* __restrict__ o, int gate, int prep) {
  constexpr int NW = kDecodeWarps, RW = DK / NW, CL = DV / 32;
  __shared__ float sq[DK], sk[DK], sa[DK], sv[DV], su[DV];
  __shared__ __align__(16) float pk[NW][DV];
  __shared__ __align__(16) float pq[NW][DV];
  __shared__ float sqk, sbeta, snorm[2];

  const size_t head = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* S = state + head * DK * DV;

  // 1. state tile of this thread: rows warp*RW .. +RW, columns lane*CL .. +CL
  float s[RW][CL];
#pragma unroll
  for (int r = 0; r < RW; ++r) Vec<CL>::load(S + (size_t)(warp * RW + r) * DV + lane * CL, s[r]);

  // 2. the token's vectors
  if (tid < DK) {
    sq[tid] = to_f32(q[head * DK + tid]);
    sk[tid] = to_f32(k[head * DK + tid]);
    sa[tid] = kGeneric ? gate_alpha(gate, prep, g + head * DK, g + head, tid) : expf(to_f32(g[head * DK + tid]));
  }
  if (tid < DV) sv[tid] = to_f32(v[head * DV + tid]);
  if (tid == 0) sbeta = kGeneric ? prep_beta(prep, to_f32(beta[head])) : to_f32(beta[head]);
  __syncthreads();
  if (kGeneric && (prep & KDA_PREP_L2NORM_QK)) {  // q, k to unit length (fused input preparation)
    if (warp < 2) {
      const float* x = warp == 0 ? sq : sk;
      float ss = 0.f;
      for (int i = lane; i < DK; i += 32) ss = fmaf(x[i], x[i], ss);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (lane == 0) snorm[warp] = rsqrtf(ss + kL2Eps);
    }
    __syncthreads();
    if (tid < DK) {
      sq[tid] *= snorm[0];
      sk[tid] *= snorm[1];
    }
    __syncthreads();
  }

  // 3. decay rows; partial column sums of S'^T k and S'^T q over this warp's rows
  float ak[CL], aq[CL];
#pragma unroll
  for (int c = 0; c < CL; ++c) ak[c] = aq[c] = 0.f;
#pragma unroll
  for (int r = 0; r < RW; ++r) {
    const int row = warp * RW + r;
    const float a = sa[row], kr = sk[row], qr = sq[row];
#pragma unroll
    for (int c = 0; c < CL; ++c) {
      s[r][c] *= a;
      ak[c] = fmaf(kr, s[r][c], ak[c]);
      aq[c] = fmaf(qr, s[r][c], aq[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < CL; ++c) {
    pk[warp][lane * CL + c] = ak[c];
    pq[warp][lane * CL + c] = aq[c];
  }
  if (warp == 0) {
    float d = 0.f;
    for (int i = lane; i < DK; i += 32) d = fmaf(sq[i], sk[i], d);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
    if (lane == 0) sqk = d;
  }
  __syncthreads();

  // 4. per column: u and the output
  if (tid < DV) {
    float ks = 0.f, qs = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      ks += pk[w][tid];
      qs += pq[w][tid];
    }
    const float u = sbeta * (sv[tid] - ks);
    su[tid] = u;
    o[head * DV + tid] = from_f32<T>(scale * fmaf(sqk, u, qs));
  }
  __syncthreads();

  // 5. rank-1 write and store
  float uc[CL];
#pragma unroll
  for (int c = 0; c < CL; ++c) uc[c] = su[lane * CL + c];
#pragma unroll
  for (int r = 0; r < RW; ++r) {
    const float kr = sk[warp * RW + r];
#pragma unroll
    for (int c = 0; c < CL; ++c) s[r][c] = fmaf(kr, uc[c], s[r][c]);
    Vec<CL>::store(S + (size_t)(warp * RW + r) * DV + lane * CL, s[r]);
  }
}

template <typename T, int DK, int DV>
cudaError_t launch_typed(const void* q, const void* k, const void* v, const void* g, const void* beta,
                         float scale, float* state, void* o, int N, int H, int gate, int prep,
                         cudaStream_t stream) {
  const unsigned heads = (unsigned)N * (unsigned)H;
  if (gate == KDA_GATE_CHANNEL && prep == 0)
    decode_step_kernel<T, DK, DV, false><<<heads, kDecodeWarps * 32, 0, stream>>>(
        (const T*)q, (const T*)k, (const T*)v, (const T*)g, (const T*)beta, scale, state, (T*)o, gate, prep);
  else
    decode_step_kernel<T, DK, DV, true><<<heads, kDecodeWarps * 32, 0, stream>>>(
        (const T*)q, (const T*)k, (const T*)v, (const T*)g, (const T*)beta, scale, state, (T*)o, gate, prep);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_dims(const void* q, const void* k, const void* v, const void* g, const void* beta,
                        float scale, float* state, void* o, int N, int H, int dk, int dv, int gate, int prep,
                        cudaStream_t stream) {
  if (dk == 128 && dv == 128) return launch_typed<T, 128, 128>(q, k, v, g, beta, scale, state, o, N, H, gate, prep, stream);
  if (dk == 128 && dv == 64) return launch_typed<T, 128, 64>(q, k, v, g, beta, scale, state, o, N, H, gate, prep, stream);
  if (dk == 64 && dv == 128) return launch_typed<T, 64, 128>(q, k, v, g, beta, scale, state, o, N, H, gate, prep, stream);
  return launch_typed<T, 64, 64>(q, k, v, g, beta, scale, state, o, N, H, gate, prep, stream);
}

}  // namespace

cudaError_t launch_decode(const void* q, const void* k, const void* v, const void* g, const void* beta,
                          float scale, float* state, void* o, int N, int H, int dk, int dv, int dtype,
                          int gate, int prep, cudaStream_t stream) {
  if (dtype == KDA_F32)
    return launch_dims<float>(q, k, v, g, beta, scale, state, o, N, H, dk, dv, gate, prep, stream);
  return launch_dims<__nv_bfloat16>(q, k, v, g, beta, scale, state, o, N, H, dk, dv, gate, prep, stream);
}

}  // namespace kda
