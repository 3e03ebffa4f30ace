// kda_backward.cu -- gradients of the KDA forward pass (token-recurrent, fp32).
//
// Given dL/do and dL/dS_T, computes dL/dq, dk, dv, dg, dbeta and dL/dS_0 by
// reverse-mode differentiation of the sequential recurrence (KimiLinear
// article, section 2.3; the scalar-gate forms of sections 2.1 and 2.2 as
// well).  One state column j evolves on its own:
//   forward:  s' = a_t .* s,  w = v_t[j] - s'.k_t,  u = beta_t w,  s = s' + k_t u,  o_t[j] = scale s.q_t
//   reverse (G = dL/dS_t[:, j]):
//     G += scale q_t dO_t[j];  dq_t += scale s_t dO_t[j]
//     du = G.k_t;  dk_t += G u;  dv_t[j] = beta_t du;  dbeta_t += du w
//     G -= beta_t k_t du;  dk_t -= beta_t s'_t du;  dg_t += G .* s'_t;  G = a_t .* G
//
// Layout of the work: one CTA per (sequence, head), 16 warps (d_v = 128) of
// 8 value columns each; lane l owns key rows RW*l .. RW*l+RW-1 (RW = d_k/32)
// of those columns, so the sums over value columns (dq, dk, dg, dbeta) stay
// inside a thread and the sums over key rows (w, du) are warp shuffles.  The
// per-token sums are added across the warps in a fixed order (deterministic).
//
// The reverse sweep needs every forward state.  Phase 1 runs the forward and
// stores the state every kCk tokens (checkpoints, workspace); phase 2 walks
// the windows of kCk tokens from the last one back: each window is re-run
// forward from its checkpoint, its decayed states s'_t written to a small
// per-CTA scratch (stays in L2), and then walked in reverse.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kCk = 16;   // tokens per checkpoint window
constexpr int kRed = 4;   // tokens per cross-warp reduction step (divides kCk)
constexpr int kColsW = 8; // value columns per warp
constexpr uint32_t kFull = 0xffffffffu;

template <typename T, int N>
__device__ __forceinline__ void load_n(const T* p, float* out) {
#pragma unroll
  for (int i = 0; i < N; ++i) out[i] = to_f32(p[i]);
}

// x[i] for a run-time i < 8 without indexing the register array.
__device__ __forceinline__ float pick8(const float (&x)[kColsW], int i) {
  float r = x[0];
#pragma unroll
  for (int j = 1; j < kColsW; ++j) r = i == j ? x[j] : r;
  return r;
}

// Sum of x over the 32 lanes, every lane gets all 8 sums.  Recursive halving:
// three exchanges of 4, 2 and 1 values (lane bits 4, 3, 2 pick the half kept)
// leave each lane one column summed over 8 lanes, two more finish that sum
// over all 32, and 8 reads gather the columns back: 17 shuffles instead of 40.
__device__ __forceinline__ void warp_allreduce8(float (&x)[kColsW]) {
  const int lane = threadIdx.x & 31;
  float a4[4], a2[2], a1;
  const bool h4 = lane & 16, h3 = lane & 8, h2 = lane & 4;
#pragma unroll
  for (int j = 0; j < 4; ++j) {  // keep columns 4*h4 .. +3, send the other half
    const float send = h4 ? x[j] : x[j + 4], keep = h4 ? x[j + 4] : x[j];
    a4[j] = keep + __shfl_xor_sync(kFull, send, 16);
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const float send = h3 ? a4[j] : a4[j + 2], keep = h3 ? a4[j + 2] : a4[j];
    a2[j] = keep + __shfl_xor_sync(kFull, send, 8);
  }
  {
    const float send = h2 ? a2[0] : a2[1], keep = h2 ? a2[1] : a2[0];
    a1 = keep + __shfl_xor_sync(kFull, send, 4);
  }
  a1 += __shfl_xor_sync(kFull, a1, 2);
  a1 += __shfl_xor_sync(kFull, a1, 1);
  // lane now holds column 4*h4 + 2*h3 + h2; column j lives in lane 4*j' where
  // bits (4,3,2) of the lane spell j
#pragma unroll
  for (int j = 0; j < kColsW; ++j) x[j] = __shfl_sync(kFull, a1, ((j >> 2) & 1) * 16 + ((j >> 1) & 1) * 8 + (j & 1) * 4);
}

struct BwdArgs {
  const void *q, *k, *v, *g, *beta, *d_o;
  const float *s0, *dsT;
  void *dq, *dk, *dv, *dg, *dbeta;
  float* ds0;
  float* ckpt;     // [CTA][NCK] state tiles of the CTA's columns, in the per-warp layout of st_tile_ws
  float* scratch;  // [CTA][kCk] decayed-state tiles, same layout
  float* part;     // split CTAs: fp32 partial dq, dk, dg [3][nsplit][tokens][DK]
  float* partb;    // split CTAs: fp32 partial dbeta, per-head dg [2][nsplit][tokens]
  float scale;
  int T, H, gate;
};

// NSPLIT CTAs share one (sequence, head), each with DV / 8 / NSPLIT warps of
// 8 columns; with NSPLIT > 1 their per-token column sums go to fp32 partial
// buffers that kda_backward_reduce_kernel adds up in split order.
template <typename IO, int DK, int DV, int NSPLIT>
__global__ void __launch_bounds__(DV / kColsW / NSPLIT * 32, 1) kda_backward_kernel(const BwdArgs a) {
  constexpr int RW = DK / 32, NW = DV / kColsW / NSPLIT;
  constexpr int TS = NW * kColsW * DK;  // floats per state tile of this CTA's columns
  static_assert(RW * 32 == DK && NW * kColsW * NSPLIT == DV, "shape");
  // dynamic shared memory: per-warp partial dq, dk, dg of kRed tokens; partial
  // dbeta and per-head dg; u_t and w_t of the window
  extern __shared__ __align__(16) float bsm[];
  auto red = reinterpret_cast<float(*)[kRed][3][DK]>(bsm);
  auto redb = reinterpret_cast<float(*)[kRed]>(bsm + NW * kRed * 3 * DK);
  auto redgh = reinterpret_cast<float(*)[kRed]>(bsm + NW * kRed * 3 * DK + NW * kRed);
  auto suw = reinterpret_cast<float(*)[2][DV]>(bsm + NW * kRed * 3 * DK + 2 * NW * kRed);
  // inputs of the current window, staged by all threads (fp32): q, k, g [kCk][DK], v, dO [kCk][DV], beta [kCk]
  float* stage = bsm + NW * kRed * 3 * DK + 2 * NW * kRed + kCk * 2 * DV;
  auto stq = reinterpret_cast<float(*)[DK]>(stage);
  auto stk = reinterpret_cast<float(*)[DK]>(stage + kCk * DK);
  auto stg = reinterpret_cast<float(*)[DK]>(stage + 2 * kCk * DK);
  auto stv = reinterpret_cast<float(*)[DV]>(stage + 3 * kCk * DK);
  auto sto = reinterpret_cast<float(*)[DV]>(stage + 3 * kCk * DK + kCk * DV);
  float* stb = stage + 3 * kCk * DK + 2 * kCk * DV;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x, bh = cta / NSPLIT, cs = cta % NSPLIT, h = bh % a.H, b = bh / a.H;
  const int T = a.T, H = a.H, gate = a.gate;
  const int r0 = RW * lane, c0 = kColsW * (cs * NW + warp);
  const int NCK = (T + kCk - 1) / kCk;
  const size_t st0 = (size_t)bh * DK * DV, ntok = (size_t)(gridDim.x / NSPLIT) * T;  // B * H * T
  float* ck = a.ckpt + (size_t)cta * NCK * TS;
  float* sc = a.scratch + (size_t)cta * kCk * TS;
  const IO* q = static_cast<const IO*>(a.q);
  const IO* k = static_cast<const IO*>(a.k);
  const IO* v = static_cast<const IO*>(a.v);
  const IO* g = static_cast<const IO*>(a.g);
  const IO* beta = static_cast<const IO*>(a.beta);
  const IO* dO = static_cast<const IO*>(a.d_o);

  auto tok_of = [&](int t) { return ((size_t)b * T + t) * H + h; };
  // stage tokens [t0, t1) of the inputs (with_q: also q and dO) into shared memory
  auto stage_window = [&](int t0, int t1, bool with_q) {
    const int n = t1 - t0, nth = NW * 32;
    for (int e = tid; e < n * DK; e += nth) {
      const int tw = e / DK, r = e % DK;
      const size_t tok = tok_of(t0 + tw);
      stk[tw][r] = to_f32(k[tok * DK + r]);
      if (with_q) stq[tw][r] = to_f32(q[tok * DK + r]);
      if (gate == KDA_GATE_CHANNEL) stg[tw][r] = expf(to_f32(g[tok * DK + r]));
    }
    for (int e = tid; e < n * DV; e += nth) {
      const int tw = e / DV, c = e % DV;
      const size_t tok = tok_of(t0 + tw);
      stv[tw][c] = to_f32(v[tok * DV + c]);
      if (with_q) sto[tw][c] = to_f32(dO[tok * DV + c]);
    }
    if (tid < n) {
      const size_t tok = tok_of(t0 + tid);
      stb[tid] = to_f32(beta[tok]);
      if (gate != KDA_GATE_CHANNEL) stg[tid][0] = gate == KDA_GATE_HEAD ? expf(to_f32(g[tok])) : 1.f;
    }
  };
  // decay factors of this lane's rows at window token tw (staged as exp(g))
  auto alpha_rows = [&](int tw, float* al) {
#pragma unroll
    for (int i = 0; i < RW; ++i) al[i] = gate == KDA_GATE_CHANNEL ? stg[tw][r0 + i] : stg[tw][0];
  };
  // 8-column tile of this lane's rows, row-major [DK][DV] with leading dimension DV
  auto st_tile = [&](float* base, const float (&x)[RW][kColsW]) {
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      float4* p = reinterpret_cast<float4*>(base + (size_t)(r0 + i) * DV + c0);
      p[0] = make_float4(x[i][0], x[i][1], x[i][2], x[i][3]);
      p[1] = make_float4(x[i][4], x[i][5], x[i][6], x[i][7]);
    }
  };
  // the same tile in the workspace's own layout: per warp, float4 number f of
  // lane l at (f * 32 + l), so each warp store or load covers 512 contiguous bytes
  auto st_tile_ws = [&](float* base, const float (&x)[RW][kColsW]) {
    float4* p = reinterpret_cast<float4*>(base) + (size_t)warp * (2 * RW * 32) + lane;
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      p[(2 * i) * 32] = make_float4(x[i][0], x[i][1], x[i][2], x[i][3]);
      p[(2 * i + 1) * 32] = make_float4(x[i][4], x[i][5], x[i][6], x[i][7]);
    }
  };
  auto ld_tile_ws = [&](const float* base, float (&x)[RW][kColsW]) {
    const float4* p = reinterpret_cast<const float4*>(base) + (size_t)warp * (2 * RW * 32) + lane;
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      const float4 lo = p[(2 * i) * 32], hi = p[(2 * i + 1) * 32];
      x[i][0] = lo.x, x[i][1] = lo.y, x[i][2] = lo.z, x[i][3] = lo.w;
      x[i][4] = hi.x, x[i][5] = hi.y, x[i][6] = hi.z, x[i][7] = hi.w;
    }
  };
  auto ld_tile = [&](const float* base, float (&x)[RW][kColsW]) {
#pragma unroll
    for (int i = 0; i < RW; ++i) {
      const float4* p = reinterpret_cast<const float4*>(base + (size_t)(r0 + i) * DV + c0);
      const float4 lo = p[0], hi = p[1];
      x[i][0] = lo.x, x[i][1] = lo.y, x[i][2] = lo.z, x[i][3] = lo.w;
      x[i][4] = hi.x, x[i][5] = hi.y, x[i][6] = hi.z, x[i][7] = hi.w;
    }
  };
  // one forward token on this lane's tile: S <- S' + k u^T, returns S' in sp, u and w
  auto fwd_token = [&](int tw, float (&S)[RW][kColsW], float (&sp)[RW][kColsW], float (&u)[kColsW],
                       float (&w)[kColsW]) {
    float al[RW], kk[RW], vv[kColsW];
    alpha_rows(tw, al);
#pragma unroll
    for (int i = 0; i < RW; ++i) kk[i] = stk[tw][r0 + i];
#pragma unroll
    for (int j = 0; j < kColsW; ++j) vv[j] = stv[tw][c0 + j];
    const float bt = stb[tw];
#pragma unroll
    for (int j = 0; j < kColsW; ++j) w[j] = 0.f;
#pragma unroll
    for (int i = 0; i < RW; ++i)
#pragma unroll
      for (int j = 0; j < kColsW; ++j) {
        sp[i][j] = al[i] * S[i][j];
        w[j] = fmaf(sp[i][j], kk[i], w[j]);
      }
    warp_allreduce8(w);
#pragma unroll
    for (int j = 0; j < kColsW; ++j) {
      w[j] = vv[j] - w[j];
      u[j] = bt * w[j];
    }
#pragma unroll
    for (int i = 0; i < RW; ++i)
#pragma unroll
      for (int j = 0; j < kColsW; ++j) S[i][j] = fmaf(kk[i], u[j], sp[i][j]);
  };

  // ---- phase 1: forward, checkpoint every kCk tokens
  float S[RW][kColsW];
#pragma unroll
  for (int i = 0; i < RW; ++i)
#pragma unroll
    for (int j = 0; j < kColsW; ++j) S[i][j] = a.s0 ? a.s0[st0 + (size_t)(r0 + i) * DV + c0 + j] : 0.f;
  for (int t0 = 0; t0 < T; t0 += kCk) {
    const int t1 = min(T, t0 + kCk);
    st_tile_ws(ck + (size_t)(t0 / kCk) * TS, S);
    __syncthreads();  // the previous tile's inputs are no longer read
    stage_window(t0, t1, false);
    __syncthreads();
    for (int t = t0; t < t1; ++t) {
      float sp[RW][kColsW], u[kColsW], w[kColsW];
      fwd_token(t - t0, S, sp, u, w);
    }
  }

  // ---- phase 2: windows in reverse
  float G[RW][kColsW];
#pragma unroll
  for (int i = 0; i < RW; ++i)
#pragma unroll
    for (int j = 0; j < kColsW; ++j) G[i][j] = a.dsT ? a.dsT[st0 + (size_t)(r0 + i) * DV + c0 + j] : 0.f;
  for (int m = NCK - 1; m >= 0; --m) {
    const int t0 = m * kCk, t1 = min(T, t0 + kCk);
    // (a) re-run the window forward from its checkpoint
    __syncthreads();  // the previous window's inputs are no longer read
    stage_window(t0, t1, true);
    __syncthreads();
    ld_tile_ws(ck + (size_t)m * TS, S);
    for (int t = t0; t < t1; ++t) {
      float sp[RW][kColsW], u[kColsW], w[kColsW];
      fwd_token(t - t0, S, sp, u, w);
      st_tile_ws(sc + (size_t)(t - t0) * TS, sp);
      if (lane < kColsW) {
        suw[t - t0][0][c0 + lane] = pick8(u, lane);
        suw[t - t0][1][c0 + lane] = pick8(w, lane);
      }
    }
    __syncwarp();
    // (b) reverse over the window in steps of kRed tokens
    for (int s1 = t1; s1 > t0; s1 = max(t0, ((s1 - 1 - t0) / kRed) * kRed + t0)) {
      const int s0 = ((s1 - 1 - t0) / kRed) * kRed + t0;  // this step: tokens [s0, s1)
      for (int t = s1 - 1; t >= s0; --t) {
        const size_t tok = tok_of(t);
        const int tw = t - t0, tr = t - s0;
        float al[RW], kk[RW], qq[RW], dd[kColsW], u[kColsW], w[kColsW], sp[RW][kColsW];
        alpha_rows(tw, al);
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          kk[i] = stk[tw][r0 + i];
          qq[i] = stq[tw][r0 + i];
        }
#pragma unroll
        for (int j = 0; j < kColsW; ++j) dd[j] = sto[tw][c0 + j];
        const float bt = stb[tw];
#pragma unroll
        for (int j = 0; j < kColsW; ++j) {
          u[j] = suw[tw][0][c0 + j];
          w[j] = suw[tw][1][c0 + j];
        }
        ld_tile_ws(sc + (size_t)tw * TS, sp);
        float pdq[RW], du[kColsW];
#pragma unroll
        for (int j = 0; j < kColsW; ++j) du[j] = 0.f;
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          pdq[i] = 0.f;
#pragma unroll
          for (int j = 0; j < kColsW; ++j) {
            const float st = fmaf(kk[i], u[j], sp[i][j]);  // S_t
            G[i][j] = fmaf(a.scale * qq[i], dd[j], G[i][j]);
            pdq[i] = fmaf(st, dd[j], pdq[i]);
            du[j] = fmaf(G[i][j], kk[i], du[j]);
          }
          pdq[i] *= a.scale;
        }
        warp_allreduce8(du);
        float pdb = 0.f;
#pragma unroll
        for (int j = 0; j < kColsW; ++j) pdb = fmaf(du[j], w[j], pdb);
        if (lane < kColsW) {
          IO* dvp = static_cast<IO*>(a.dv);
          dvp[tok * DV + c0 + lane] = from_f32<IO>(bt * pick8(du, lane));
        }
        float pdk[RW], pdg[RW];
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          pdk[i] = 0.f;
          pdg[i] = 0.f;
#pragma unroll
          for (int j = 0; j < kColsW; ++j) {
            pdk[i] = fmaf(G[i][j], u[j], pdk[i]);
            pdk[i] = fmaf(-bt * sp[i][j], du[j], pdk[i]);
            G[i][j] = fmaf(-bt * kk[i], du[j], G[i][j]);
            pdg[i] = fmaf(G[i][j], sp[i][j], pdg[i]);
            G[i][j] *= al[i];
          }
        }
#pragma unroll
        for (int i = 0; i < RW; ++i) {
          red[warp][tr][0][r0 + i] = pdq[i];
          red[warp][tr][1][r0 + i] = pdk[i];
          red[warp][tr][2][r0 + i] = pdg[i];
        }
        if (gate == KDA_GATE_HEAD) {  // the per-head gate's gradient sums all key rows
          float x = 0.f;
#pragma unroll
          for (int i = 0; i < RW; ++i) x += pdg[i];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(kFull, x, off);
          if (lane == 0) redgh[warp][tr] = x;
        }
        if (lane == 0) redb[warp][tr] = pdb;
      }
      __syncthreads();
      // sum the warps' partials in warp order and write this step's tokens
      const int nt = s1 - s0;
      for (int e = tid; e < nt * 3 * DK; e += NW * 32) {
        const int tr = e / (3 * DK), which = (e / DK) % 3, r = e % DK;
        if (which == 2 && gate != KDA_GATE_CHANNEL) continue;
        float x = 0.f;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) x += red[ww][tr][which][r];
        if (NSPLIT == 1) {
          IO* out = static_cast<IO*>(which == 0 ? a.dq : which == 1 ? a.dk : a.dg);
          out[tok_of(s0 + tr) * DK + r] = from_f32<IO>(x);
        } else {
          a.part[((size_t)which * NSPLIT + cs) * ntok * DK + tok_of(s0 + tr) * DK + r] = x;
        }
      }
      if (tid < nt) {
        float x = 0.f, y = 0.f;
#pragma unroll
        for (int ww = 0; ww < NW; ++ww) {
          x += redb[ww][tid];
          y += redgh[ww][tid];
        }
        if (NSPLIT == 1) {
          static_cast<IO*>(a.dbeta)[tok_of(s0 + tid)] = from_f32<IO>(x);
          if (gate == KDA_GATE_HEAD) static_cast<IO*>(a.dg)[tok_of(s0 + tid)] = from_f32<IO>(y);
        } else {
          a.partb[(size_t)cs * ntok + tok_of(s0 + tid)] = x;
          a.partb[((size_t)NSPLIT + cs) * ntok + tok_of(s0 + tid)] = y;
        }
      }
      __syncthreads();
    }
  }
  if (a.ds0) st_tile(a.ds0 + st0, G);
}

// Sums the NSPLIT partials of dq, dk, dg (per channel) and dbeta, dg (per
// head) in split order and writes them in the output type.
template <typename IO>
__global__ void kda_backward_reduce_kernel(const BwdArgs a, size_t ntok, int DK, int nsplit) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x, n = ntok * DK;
  if (i < n) {
    for (int which = 0; which < 3; ++which) {
      if (which == 2 && a.gate != KDA_GATE_CHANNEL) continue;
      float x = 0.f;
      for (int s = 0; s < nsplit; ++s) x += a.part[((size_t)which * nsplit + s) * n + i];
      static_cast<IO*>(which == 0 ? a.dq : which == 1 ? a.dk : a.dg)[i] = from_f32<IO>(x);
    }
  }
  if (i < ntok) {
    float x = 0.f, y = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      x += a.partb[(size_t)s * ntok + i];
      y += a.partb[((size_t)nsplit + s) * ntok + i];
    }
    static_cast<IO*>(a.dbeta)[i] = from_f32<IO>(x);
    if (a.gate == KDA_GATE_HEAD) static_cast<IO*>(a.dg)[i] = from_f32<IO>(y);
  }
}

template <int DK, int DV, int NSPLIT>
constexpr size_t smem_bytes() {
  constexpr int NW = DV / kColsW / NSPLIT;
  return sizeof(float) * ((size_t)NW * kRed * 3 * DK + 2 * NW * kRed + (size_t)kCk * 2 * DV +
                          (size_t)kCk * (3 * DK + 2 * DV + 1));
}

template <typename IO, int DK, int DV, int NSPLIT>
cudaError_t launch_split(const BwdArgs& a, int BH, cudaStream_t stream) {
  constexpr size_t smem = smem_bytes<DK, DV, NSPLIT>();
  cudaError_t e = cudaFuncSetAttribute(kda_backward_kernel<IO, DK, DV, NSPLIT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kda_backward_kernel<IO, DK, DV, NSPLIT><<<BH * NSPLIT, DV / kColsW / NSPLIT * 32, smem, stream>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || NSPLIT == 1) return e;
  const size_t ntok = (size_t)BH * a.T, n = ntok * DK;
  kda_backward_reduce_kernel<IO><<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(a, ntok, DK, NSPLIT);
  return cudaGetLastError();
}

template <typename IO, int DK, int DV>
cudaError_t launch_typed(const BwdArgs& a, int BH, int nsplit, cudaStream_t stream) {
  if (nsplit == 4) return launch_split<IO, DK, DV, 4>(a, BH, stream);
  if (nsplit == 2) return launch_split<IO, DK, DV, 2>(a, BH, stream);
  return launch_split<IO, DK, DV, 1>(a, BH, stream);
}

template <typename IO>
cudaError_t launch_dims(const BwdArgs& a, int BH, int dk, int dv, int nsplit, cudaStream_t stream) {
  if (dk == 128 && dv == 128) return launch_typed<IO, 128, 128>(a, BH, nsplit, stream);
  if (dk == 128 && dv == 64) return launch_typed<IO, 128, 64>(a, BH, nsplit, stream);
  if (dk == 64 && dv == 128) return launch_typed<IO, 64, 128>(a, BH, nsplit, stream);
  return launch_typed<IO, 64, 64>(a, BH, nsplit, stream);
}

// CTAs per (sequence, head): more when few pairs would leave SMs idle (up to
// 4 and one wave of a 148-SM part); a fixed function of the shape.
int backward_split(int BH) {
  int n = 1;
  while (n < 4 && BH * n * 2 <= 148) n *= 2;
  return n;
}

}  // namespace

size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv) {
  const size_t nck = ((size_t)T + kCk - 1) / kCk, ntok = (size_t)B * T * H;
  const int ns = backward_split(B * H);
  const size_t part = ns > 1 ? (size_t)ns * ntok * (3 * (size_t)dk + 2) : 0;
  return ((size_t)B * H * (nck + kCk) * dk * dv + part) * sizeof(float);
}

cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* g, const void* beta,
                            float scale, const float* s0, const void* d_o, const float* dsT, void* dq, void* dk_out,
                            void* dv_out, void* dg, void* dbeta, float* ds0, int B, int T, int H, int dk, int dv,
                            int dtype, int gate, void* ws, cudaStream_t stream) {
  const size_t nck = ((size_t)T + kCk - 1) / kCk;
  BwdArgs a;
  a.q = q, a.k = k, a.v = v, a.g = g, a.beta = beta, a.d_o = d_o;
  a.s0 = s0, a.dsT = dsT;
  a.dq = dq, a.dk = dk_out, a.dv = dv_out, a.dg = dg, a.dbeta = dbeta, a.ds0 = ds0;
  const int ns = backward_split(B * H);
  const size_t ntok = (size_t)B * T * H;
  a.ckpt = static_cast<float*>(ws);
  a.scratch = a.ckpt + (size_t)B * H * nck * dk * dv;
  a.part = a.scratch + (size_t)B * H * kCk * dk * dv;
  a.partb = a.part + (size_t)ns * ntok * 3 * dk;
  a.scale = scale, a.T = T, a.H = H, a.gate = gate;
  if (dtype == KDA_F32) return launch_dims<float>(a, B * H, dk, dv, ns, stream);
  return launch_dims<__nv_bfloat16>(a, B * H, dk, dv, ns, stream);
}

}  // namespace kda
