// kda_backward_chunk.cu -- gradients of the KDA forward pass in the chunkwise form.
//
// Differentiates the chunk equations of the forward (KimiLinear article,
// section 2.3 for the recurrence, section 3.1 for the chunkwise algorithm and
// section 3.2 for the per-chunk C x C score matrices).  One chunk of C = 64
// tokens with entering state S0 (d_k x d_v), G_i the in-chunk inclusive
// cumsum of the log-gates, Gamma_i = exp(G_i), gamma = Gamma_C:
//
//   Q+ = scale q . Gamma,  K+ = k . Gamma,  Kbar_j = k_j . Gamma_C / Gamma_j
//   P  = strict_tril(K+ K-^T)  with K- = k / Gamma     (pairwise: sum_r k_ir k_jr exp(G_ir - G_jr))
//   Aqk = tril(Q+ K-^T),  T = (I + diag(beta) P)^-1,  W = T diag(beta) K+,  U = T diag(beta) V
//   V' = U - W S0,  O = Q+ S0 + Aqk V',  S1 = diag(gamma) S0 + Kbar^T V'
//
// Reverse mode, chunk by chunk from the last one, with dS = dL/dS1:
//
//   dV' = Aqk^T dO + Kbar dS                       dS0 = diag(gamma) dS + Q+^T dO - W^T dV'
//   dAqk = tril(dO V'^T)   dQ+ = dO S0^T + dAqk K-   dKbar = V' dS^T   dgamma = rowsum(dS . S0)
//   dW = -dV' S0^T   dU = dV'   dT = dU (beta V)^T + dW (beta K+)^T   dA = -T^T dT T^T (strictly lower)
//   dv = beta . T^T dU,   dK+ = beta . T^T dW + (beta dA) K-,   dK- = dAqk^T Q+ + (beta dA)^T K+
//   dbeta = rowsum(V . T^T dU) + rowsum(K+ . T^T dW) + rowsum(dA . P)
//
// and the factors are folded back into dq, dk and dG, whose reverse in-chunk
// cumsum is dg.  The pairwise products use factored operands relative to the
// chunk's token 31 (K+_r = k exp(G - G_31), K-_r = k exp(G_31 - G)); their
// products are independent of that reference, so the reference is a constant
// for differentiation.  A chunk whose cumulative gates leave +-kSpan of the
// reference takes an exact per-element path instead (exp of each difference).
//
// Four launches per group of (sequence, head) pairs (as many as the workspace
// holds), the last three chained to the one before by programmatic dependent
// launch:
//   1. bwd_prep    (chunk, seq x head): W, U, Q+, Kbar, Aqk, P, T, gamma per
//      chunk; for bf16 at d_k = d_v = 128 from 16 (sequence, head) pairs on,
//      the prefill's tcgen05 preparation kernel in its backward mode
//   2. bwd_pass    (seq x head x column slice, 2 roles): the forward state
//      replay (checkpoints S0 and V' per chunk) and the reverse dS sweep
//      (dS and dV' per chunk, dL/dS_0); the columns of the state evolve
//      independently in both; with the tcgen05 preparation, one CTA per
//      (sequence, head) and role on the tcgen05 tensor cores, the state in
//      tensor memory
//   3. bwd_local_a (chunk, seq x head): the products contracting over d_v:
//      dAqk, dT (first part), dv, dbeta (first part), dO S0^T, dW, dKbar, dgamma
//   4. bwd_local_b (chunk, seq x head): the rest, and dq, dk, dg, dbeta
// Arithmetic of the per-chunk kernels here: warp-level tensor-core products
// (mma.sync), fp32 accumulation.
// fp32 inputs: fp32 shared tiles, m16n8k8 with tf32 operands in the
// three-term split (a_hi b_hi + a_hi b_lo + a_lo b_hi), which keeps fp32-level
// accuracy; fp32 workspace.  bf16 inputs: bf16 operand images (ldmatrix, with
// .trans where the stored rows run along the other index), m16n8k16 with bf16
// operands; the state passes keep the state in fp32 registers and read each
// chunk's operands as one bf16 record; the decay factors, the fold into the
// gradients and every sum stay fp32.  No atomics: every sum runs in a fixed
// order, so results are bit-reproducible.
#include <cudaTypedefs.h>

#include <algorithm>
#include <type_traits>

#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

constexpr int kC = 64;          // tokens per chunk
constexpr int kRef = 31;        // reference token of the factored pairwise operands
constexpr float kSpan = 64.f;   // factored operands need |G_i - G_ref| <= kSpan in every channel
constexpr int kThreads = 512;   // 16 warps in the per-chunk kernels
constexpr int kWarps = kThreads / 32;
constexpr int kPassThreads = 256;  // 8 warps in the state passes (longer tiles, fewer loads per MMA)
constexpr int kLC = kC + 4;     // leading dimension of the C x C shared tiles

// ------------------------------------------------------------------ launch chaining
// The four kernels of a call are chained by programmatic dependent launch:
// each kernel lets the next one be scheduled as soon as all of its CTAs have
// started (so the next grid's CTAs fill the SMs its last wave frees), and the
// next one waits for the whole previous grid, memory included, before its
// first access.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------------ warp MMA
__device__ __forceinline__ uint32_t tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// A strided fp32 matrix view in shared memory: element (i, j) at p[i*rs + j*cs].
struct View {
  const float* p;
  int rs, cs;
  __device__ __forceinline__ float at(int i, int j) const { return p[i * rs + j * cs]; }
};
__device__ __forceinline__ View rowm(const float* p, int ld) { return View{p, ld, 1}; }  // X
__device__ __forceinline__ View colm(const float* p, int ld) { return View{p, 1, ld}; }  // X^T

// acc[MT][NT] (a (16 MT) x (8 NT) tile at rows m0, columns n0) += A[m0.., 0:K] B[0:K, n0..].
// Fragment layout of mma.m16n8k8: g = lane / 4, t = lane % 4; A holds (g, t),
// (g+8, t), (g, t+4), (g+8, t+4); B holds (t, g), (t+4, g); the accumulator
// holds rows g, g+8 and columns 2t, 2t+1.  X3: three-term tf32 split.
template <int MT, int NT, bool X3, int K>
__device__ __forceinline__ void warp_mma(float (&acc)[MT][NT][4], View A, View B, int m0, int n0) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int k0 = 0; k0 < K; k0 += 8) {
    uint32_t ah[MT][4], al[MT][4], bh[NT][2], bl[NT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int r = m0 + 16 * mt + g;
      const float x[4] = {A.at(r, k0 + t), A.at(r + 8, k0 + t), A.at(r, k0 + t + 4), A.at(r + 8, k0 + t + 4)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ah[mt][e] = tf32_rna(x[e]);
        if (X3) al[mt][e] = tf32_rna(x[e] - __uint_as_float(ah[mt][e]));
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int c = n0 + 8 * nt + g;
      const float y[2] = {B.at(k0 + t, c), B.at(k0 + t + 4, c)};
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        bh[nt][e] = tf32_rna(y[e]);
        if (X3) bl[nt][e] = tf32_rna(y[e] - __uint_as_float(bh[nt][e]));
      }
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (X3) {
          mma_tf32(acc[mt][nt], al[mt][0], al[mt][1], al[mt][2], al[mt][3], bh[nt][0], bh[nt][1]);
          mma_tf32(acc[mt][nt], ah[mt][0], ah[mt][1], ah[mt][2], ah[mt][3], bl[nt][0], bl[nt][1]);
        }
        mma_tf32(acc[mt][nt], ah[mt][0], ah[mt][1], ah[mt][2], ah[mt][3], bh[nt][0], bh[nt][1]);
      }
  }
}

// The same product for K-contiguous operands: A is [M][lda] and B^T is [N][ldb]
// (element (k, n) of B at B[n*ldb + k]), both with k contiguous.  Fragments
// come from ldmatrix (8 x 8 b16 matrices = 8 rows x 4 fp32): one x4 per A tile
// and one x4 per pair of B tiles.  Row starts must be 16-byte aligned; ld = 4
// (mod 32) floats keeps the 8 rows of each matrix in distinct bank groups.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const float* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const float* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
template <int MT, int NT, bool X3, int K>
__device__ __forceinline__ void warp_mma_kk(float (&acc)[MT][NT][4], const float* A, int lda, const float* B, int ldb,
                                            int m0, int n0) {
  const int lane = threadIdx.x & 31, mat = lane >> 3, rr = lane & 7;
  // odd NT: the last B tile by an x2 load (lanes 0-15 give its row addresses)
  const float* pb1 = B + (n0 + 8 * (NT - 1) + rr) * ldb + 4 * (mat & 1);
  // this lane's row address in each x4 load
  const float* pa = A + (m0 + rr + 8 * (mat & 1)) * lda + 4 * (mat >> 1);
  const float* pb = B + (n0 + rr + 8 * (mat >> 1)) * ldb + 4 * (mat & 1);
#pragma unroll
  for (int k0 = 0; k0 < K; k0 += 8) {
    uint32_t ah[MT][4], al[MT][4], bh[NT][2], bl[NT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      uint32_t r[4];
      ldsm_x4(r, pa + 16 * mt * lda + k0);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x = __uint_as_float(r[e]);
        ah[mt][e] = tf32_rna(x);
        if (X3) al[mt][e] = tf32_rna(x - __uint_as_float(ah[mt][e]));
      }
    }
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      uint32_t r[4];
      ldsm_x4(r, pb + 16 * np * ldb + k0);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x = __uint_as_float(r[e]);
        const int nt = 2 * np + (e >> 1), h = e & 1;
        bh[nt][h] = tf32_rna(x);
        if (X3) bl[nt][h] = tf32_rna(x - __uint_as_float(bh[nt][h]));
      }
    }
    if constexpr (NT % 2 == 1) {
      uint32_t r[2];
      ldsm_x2(r, pb1 + k0);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float x = __uint_as_float(r[h]);
        bh[NT - 1][h] = tf32_rna(x);
        if (X3) bl[NT - 1][h] = tf32_rna(x - __uint_as_float(bh[NT - 1][h]));
      }
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (X3) {
          mma_tf32(acc[mt][nt], al[mt][0], al[mt][1], al[mt][2], al[mt][3], bh[nt][0], bh[nt][1]);
          mma_tf32(acc[mt][nt], ah[mt][0], ah[mt][1], ah[mt][2], ah[mt][3], bl[nt][0], bl[nt][1]);
        }
        mma_tf32(acc[mt][nt], ah[mt][0], ah[mt][1], ah[mt][2], ah[mt][3], bh[nt][0], bh[nt][1]);
      }
  }
}

// Split of an R x N output over NW warps: WM x WN warps, each (16 MT) x (8 NT).
template <int R, int N, int NW = kWarps>
struct Tiling {
  static constexpr int WM = (R / 16 >= NW) ? NW : R / 16;
  static constexpr int WN = NW / WM;
  static constexpr int MT = R / 16 / WM;
  static constexpr int NT = N / 8 / WN;
  static_assert(WM * WN == NW && MT * 16 * WM == R && NT * 8 * WN == N, "tiling");
  __device__ static int m0(int warp) { return (warp % WM) * MT * 16; }
  __device__ static int n0(int warp) { return (warp / WM) * NT * 8; }
};

template <int MT, int NT>
__device__ __forceinline__ void zero(float (&acc)[MT][NT][4]) {
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
}
// f(mt, nt, e, row, col) over the accumulator elements acc[mt][nt][e] of this lane.
template <int MT, int NT, typename F>
__device__ __forceinline__ void for_acc(int m0, int n0, F&& f) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) f(mt, nt, e, m0 + 16 * mt + g + 8 * (e >> 1), n0 + 8 * nt + 2 * t + (e & 1));
}

// Per-row sums of a tile product: each lane adds to rp[mt][half] for its rows
// m0 + 16 mt + g + 8 half; the 4 lanes of a row are then combined and lane
// t = 0 writes the warp's row sums to out[row] (one slot per column group).
template <int MT>
__device__ __forceinline__ void row_sums_out(float (&rp)[MT][2], int m0, float* out) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float x = rp[mt][hh];
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      if (t == 0) out[m0 + 16 * mt + g + 8 * hh] = x;
    }
}

// ------------------------------------------------------------------ tiles
// Rows of one chunk of a [B, T, H, len] tensor: token i of chunk (b, t0) is
// row ((b*T + t0 + i) * H + h).  Loads columns col0 .. col0+W-1 of its 64 rows
// as fp32 into dst (leading dimension ld), rows >= nv as zeros, times mult[i]
// when mult is given.
template <typename IO, int W>
__device__ __forceinline__ void load_rows(float* dst, int ld, const IO* src, size_t row0, int H, int nv, int len,
                                          int col0, const float* mult = nullptr) {
  constexpr int V = 16 / sizeof(IO);  // elements per 16-byte load
  constexpr int PER_ROW = W / V, N = kC * PER_ROW, IT = (N + kThreads - 1) / kThreads;
  uint4 w[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {  // all loads in flight before the first store
    const int idx = threadIdx.x + it * kThreads, i = idx / PER_ROW, c = (idx % PER_ROW) * V;
    w[it] = (idx < N && i < nv) ? __ldg(reinterpret_cast<const uint4*>(src + (row0 + (size_t)i * H) * len + col0 + c))
                                : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const int idx = threadIdx.x + it * kThreads, i = idx / PER_ROW, c = (idx % PER_ROW) * V;
    if (idx >= N) break;
    float x[V];
    if constexpr (std::is_same<IO, float>::value) {
      x[0] = __uint_as_float(w[it].x), x[1] = __uint_as_float(w[it].y), x[2] = __uint_as_float(w[it].z),
      x[3] = __uint_as_float(w[it].w);
    } else {
      const uint32_t u[4] = {w[it].x, w[it].y, w[it].z, w[it].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
        x[2 * e] = f.x, x[2 * e + 1] = f.y;
      }
    }
    if (mult) {
      const float m = mult[i];
#pragma unroll
      for (int e = 0; e < V; ++e) x[e] *= m;
    }
#pragma unroll
    for (int e = 0; e < V; e += 4)
      *reinterpret_cast<float4*>(dst + i * ld + c + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
  }
}
// Asynchronous 16-byte copies global -> shared (cp.async); cp_wait() waits
// for all of this thread's copies, a barrier then publishes them.
__device__ __forceinline__ void cp_async16(float* dst, const float* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// 16-byte cp.async of which the first `bytes` (0 or 16) come from src, the rest zero-filled.
__device__ __forceinline__ void cp16(void* dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(bytes)
               : "memory");
}
// fp32 rows x cols block from global (leading dimension gld) into shared (ld),
// cols % 4 == 0, by cp.async: complete after cp_wait().
template <int NTH = kThreads>
__device__ __forceinline__ void load_f32(float* dst, int ld, const float* src, int gld, int rows, int cols) {
  const int per = cols / 4;
  for (int idx = threadIdx.x; idx < rows * per; idx += NTH) {
    const int i = idx / per, c = (idx % per) * 4;
    cp_async16(dst + i * ld + c, src + (size_t)i * gld + c);
  }
}
template <int NTH = kThreads>
__device__ __forceinline__ void store_f32(float* dst, int gld, const float* src, int ld, int rows, int cols) {
  const int per = cols / 4;
  for (int idx = threadIdx.x; idx < rows * per; idx += NTH) {
    const int i = idx / per, c = (idx % per) * 4;
    *reinterpret_cast<float4*>(dst + (size_t)i * gld + c) = *reinterpret_cast<const float4*>(src + i * ld + c);
  }
}

// Per-channel log-gates of one chunk into sG [64][ld] (zeros past nv): per
// channel, per head (broadcast over the channels) or none; then the inclusive
// cumsum over the tokens, in place (one thread per channel, the column in
// registers).  Returns (block-uniform) whether the chunk needs the exact
// pairwise path: some |G_i - G_ref| above kSpan.
template <typename IO, int DK>
__device__ __forceinline__ bool load_gates_cumsum(float* sG, int ld, const IO* g, int gate, size_t row0, int H,
                                                  int nv) {
  if (gate == KDA_GATE_CHANNEL) {
    load_rows<IO, DK>(sG, ld, g, row0, H, nv, DK, 0);
  } else {
    for (int idx = threadIdx.x; idx < kC * DK; idx += kThreads) {
      const int i = idx / DK, r = idx % DK;
      sG[i * ld + r] = (gate == KDA_GATE_HEAD && i < nv) ? to_f32(g[row0 + (size_t)i * H]) : 0.f;
    }
  }
  __syncthreads();
  bool bad = false;
  if (threadIdx.x < DK) {
    float x[kC];
#pragma unroll
    for (int i = 0; i < kC; ++i) x[i] = sG[i * ld + threadIdx.x];
#pragma unroll
    for (int i = 1; i < kC; ++i) x[i] += x[i - 1];
#pragma unroll
    for (int i = 0; i < kC; ++i) {
      sG[i * ld + threadIdx.x] = x[i];
      bad |= !(fabsf(x[i] - x[kRef]) <= kSpan);
    }
  }
  return __syncthreads_or(bad) != 0;
}

// ------------------------------------------------------------------ arguments
struct ChunkBwdArgs {
  const void *q, *k, *v, *g, *beta, *d_o;
  const float *s0, *dsT;
  void *dq, *dk, *dv, *dg, *dbeta;
  float* ds0;
  float *dq32, *dk32;  // bf16 inputs: when set, dq and dk go here in fp32 instead (for a later chain rule)
  float scale;
  int T, H, NC, gate;
  int bh0;  // first (sequence, head) of this launch group: bh = bh0 + local index
  int tc_rec;  // bf16, d_k = d_v = 128: the pass record in the tensor-core passes' layout (TcRec)
  // workspace (fp32), record rec = (bh - bh0) * NC + chunk
  float *W, *U, *Qp, *Kb;  // [rec][64][d_k] (U: [64][d_v]): W, U, Q+, Kbar
  float *Wt, *Qpt, *Kbt;   // [rec][d_k][64]: their transposes for the state passes (fp32 inputs)
  float *Aqk, *Tm, *Pkk;   // [rec][64][64]: Aqk^T (transposed; fp32 inputs), T, P
  __nv_bfloat16* prec;     // bf16 inputs: [rec] bf16 pass record (W, W^T, Kbar, Kbar^T, Q+^T, Aqk^T)
  float* gam;              // [rec][d_k]: gamma
  float *S0c, *dSc;        // [rec][d_k][d_v]: state entering the chunk, dL/d(state leaving it)
  float *Vp, *dVp;         // [rec][64][d_v]: V', dV'
  float *dAqk, *dT1;       // [rec][64][64]: dAqk, dU (beta V)^T (strictly lower)
  float *dQs, *dW, *dKb;   // [rec][64][d_k]: dO S0^T, dW, dKbar
  float* dgam;             // [rec][d_k]: rowsum(dS . S0)
  float* dbu;              // [rec][64]: rowsum(V . T^T dU)
};

__device__ __forceinline__ size_t row_of(const ChunkBwdArgs& a, int bh, int t0) {
  return ((size_t)(bh / a.H) * a.T + t0) * a.H + bh % a.H;
}

// Element offsets of the bf16 pass record of one chunk (bf16 inputs): the
// state passes' operands in their shared-memory layout, rows padded by 16
// bytes.  The passes read the operands they need transposed (Aqk^T, Q+^T,
// W^T, Kbar^T) with ldmatrix.trans, so each is stored once, row-major.
using bf16 = __nv_bfloat16;
template <int DK>
struct PassRec {  // element offsets of the bf16 pass record of one chunk (all row-major)
  static constexpr int LKb = DK + 8, LCb = kC + 8;
  static constexpr int oAqk = 0;                 // [64][LCb]  Aqk        (reverse sweep, read transposed)
  static constexpr int oQp = oAqk + kC * LCb;    // [64][LKb]  Q+         (reverse sweep, read transposed)
  static constexpr int oW = oQp + kC * LKb;      // [64][LKb]  W          (both; transposed in the reverse sweep)
  static constexpr int oKb = oW + kC * LKb;      // [64][LKb]  Kbar       (both; transposed in the forward replay)
  static constexpr int n = oKb + kC * LKb;       // the reverse sweep reads [0, n), the forward replay [oW, n)
  static_assert(oQp % 8 == 0 && oW % 8 == 0 && oKb % 8 == 0 && n % 8 == 0, "16 B");
};

// With d_k = d_v = 128 the state passes run on the tcgen05 tensor cores and
// read the record as the canonical 128-byte-swizzled token-row tiles of
// their MMA operands (the layout a TMA tile load of [64 tokens][64 channels]
// produces): element (token i, channel c) of a 64 x 128 tile at byte
// (c / 64) * 8192 + i * 128 + (((c % 64) / 8) ^ (i % 8)) * 16 + (c % 8) * 2.
// Byte offsets inside the record (the record keeps PassRec's stride):
struct TcRec {
  static constexpr uint32_t oW = kTcRecW;      // W    [64 tokens][128 channels]
  static constexpr uint32_t oQp = kTcRecQp;    // Q+   [64 tokens][128 channels]
  static constexpr uint32_t oKb = kTcRecKb;    // Kbar [64 tokens][128 channels]
  static constexpr uint32_t oAqk = kTcRecAqk;  // Aqk  [64 query tokens i][64 key tokens j]
  static constexpr uint32_t bytes = kTcRecBytes;
};
static_assert(TcRec::bytes <= PassRec<128>::n * 2, "the tensor-core record fits the record stride");
template <int DK, int DV>
constexpr bool kTcPass = DK == 128 && DV == 128;
__device__ __forceinline__ uint32_t tile_off(int i, int c) {  // byte offset of (token i, channel c) in a 64-row tile
  return (uint32_t)((c >> 6) * 8192 + i * 128 + ((((c & 63) >> 3) ^ (i & 7)) << 4) + (c & 7) * 2);
}

// T = (I + diag(beta) P)^-1 for a strictly lower 64 x 64 P (fp32, leading
// dimension kLC) by 16 x 16 blocks, on the NT first threads of the block
// (named barrier 1): the diagonal blocks by forward substitution (one thread
// per block column, the column in registers), then the blocks below the
// diagonal level by level, T_IJ = -T_II (sum_{K=J..I-1} A_IK T_KJ) with
// A = diag(beta) P.  T (fp32, leading dimension kLC) is unit lower triangular
// with zeros above; X is a 3 x 16 x 16 fp32 scratch.
template <int NT>
__device__ __forceinline__ void bar_nt() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }
template <int NT>
__device__ __forceinline__ void solve_T_blocked(const float* sP, const float* sb, float* T, float* X, int t) {
  static_assert(NT > kC && NT % 32 == 0, "threads");
  if (t < kC) {  // diagonal block I = t / 16, column jj = t % 16
    const int I = t >> 4, jj = t & 15, r0 = 16 * I;
    float tc[16];
#pragma unroll
    for (int ii = 0; ii < 16; ++ii) {
      float s = 0.f;
#pragma unroll
      for (int m = 0; m < ii; ++m) s = fmaf(sP[(r0 + ii) * kLC + r0 + m], tc[m], s);
      tc[ii] = ii == jj ? 1.f : (ii < jj ? 0.f : -sb[r0 + ii] * s);
      T[(r0 + ii) * kLC + r0 + jj] = tc[ii];
    }
  } else {  // the six blocks above the diagonal are zero
    for (int e = t - kC; e < 6 * 256; e += NT - kC) {
      const int blk = e >> 8, a = (e >> 4) & 15, b = e & 15;
      const int I = blk < 3 ? 0 : (blk < 5 ? 1 : 2), J = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
      T[(16 * I + a) * kLC + 16 * J + b] = 0.f;
    }
  }
  bar_nt<NT>();
  for (int d = 1; d < 4; ++d) {
    const int nb = 4 - d;  // blocks (I, J = I - d), J = 0 .. nb-1
    for (int e = t; e < nb * 256; e += NT) {
      const int J = e >> 8, I = J + d, a = (e >> 4) & 15, b = e & 15;
      float s = 0.f;
      for (int K = J; K < I; ++K)
#pragma unroll
        for (int m = 0; m < 16; ++m) s = fmaf(sP[(16 * I + a) * kLC + 16 * K + m], T[(16 * K + m) * kLC + 16 * J + b], s);
      X[e] = sb[16 * I + a] * s;
    }
    bar_nt<NT>();
    for (int e = t; e < nb * 256; e += NT) {
      const int J = e >> 8, I = J + d, a = (e >> 4) & 15, b = e & 15;
      float s = 0.f;
#pragma unroll
      for (int m = 0; m < 16; ++m) s = fmaf(T[(16 * I + a) * kLC + 16 * I + m], X[J * 256 + m * 16 + b], s);
      T[(16 * I + a) * kLC + 16 * J + b] = -s;
    }
    bar_nt<NT>();
  }
}
constexpr int kSolveThreads = 256;  // 8 warps solve T while the others prepare the W/U operands

// ------------------------------------------------------------------ kernel 1
template <int DK, int DV>
constexpr size_t prep_smem() {
  constexpr int LK = DK + 4, LM = (DK > DV ? DK : DV) + 4;
  return sizeof(float) * ((size_t)4 * kC * LK + (size_t)kC * LM + 3 * kC * kLC + kC + DK + 3 * 256);
}

// Per chunk, fp32 inputs (IO = float; bf16 inputs take the kernels on bf16
// operands below): G, the factored and absolute operands, P and Aqk, T, W and U.
template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1) bwd_prep_kernel(const ChunkBwdArgs a) {
  pdl_trigger();
  constexpr bool X3 = std::is_same<IO, float>::value;
  constexpr int LK = DK + 4, LM = (DK > DV ? DK : DV) + 4;
  extern __shared__ __align__(16) float sm[];
  float* sG = sm;             // [64][LK] cumulative log-gates
  float* sK = sG + kC * LK;   // [64][LK] k
  float* sQ = sK + kC * LK;   // [64][LK] q, then Q+_r (fast path)
  float* sX = sQ + kC * LK;   // [64][LK] K+_r (exact path: K+), then beta K+
  float* sY = sX + kC * LK;   // [64][LM] K-_r, then beta v
  float* sP = sY + kC * LM;   // [64][kLC] P
  float* sA = sP + kC * kLC;  // [64][kLC] Aqk
  float* sT = sA + kC * kLC;  // [64][kLC] T
  float* sb = sT + kC * kLC;  // [64] beta
  float* se = sb + kC;        // [DK] exp(G_ref)
  float* sXs = se + DK;       // [3][16][16] solve scratch
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n = blockIdx.x % a.NC, lb = blockIdx.x / a.NC, bh = a.bh0 + lb, t0 = n * kC, nv = min(kC, a.T - t0);
  const size_t row0 = row_of(a, bh, t0), rec = (size_t)lb * a.NC + n;
  const IO* q = static_cast<const IO*>(a.q);
  const IO* k = static_cast<const IO*>(a.k);
  const IO* beta = static_cast<const IO*>(a.beta);

  load_rows<IO, DK>(sK, LK, k, row0, a.H, nv, DK, 0);
  load_rows<IO, DK>(sQ, LK, q, row0, a.H, nv, DK, 0);
  if (tid < kC) sb[tid] = tid < nv ? to_f32(beta[row0 + (size_t)tid * a.H]) : 0.f;
  const bool slow = load_gates_cumsum<IO, DK>(sG, LK, static_cast<const IO*>(a.g), a.gate, row0, a.H, nv);
  if (tid < DK) {
    se[tid] = expf(sG[kRef * LK + tid]);
    a.gam[rec * DK + tid] = expf(sG[(kC - 1) * LK + tid]);
  }
  for (int idx = tid; idx < kC * DK; idx += kThreads) {  // Q+^T and Kbar^T (the same values as Q+, Kbar below)
    const int r = idx / kC, i = idx % kC;
    const float G = sG[i * LK + r], qq = a.scale * sQ[i * LK + r];
    const float qp = qq * expf(G), kb = sK[i * LK + r] * expf(sG[(kC - 1) * LK + r] - G);
    a.Qpt[rec * kC * DK + idx] = qp;
    a.Kbt[rec * kC * DK + idx] = kb;
  }
  float* Qp = a.Qp + rec * kC * DK;
  float* Kb = a.Kb + rec * kC * DK;
  __syncthreads();  // sQ is rewritten in place below
  for (int idx = tid; idx < kC * DK; idx += kThreads) {
    const int i = idx / DK, r = idx % DK;
    const float G = sG[i * LK + r], kk = sK[i * LK + r], qq = a.scale * sQ[i * LK + r];
    const float gm = expf(G);
    Qp[i * DK + r] = qq * gm;
    Kb[i * DK + r] = kk * expf(sG[(kC - 1) * LK + r] - G);
    if (!slow) {
      const float d = G - sG[kRef * LK + r];
      const float ex = expf(d);
      sX[i * LK + r] = kk * ex;
      sY[i * LK + r] = kk * expf(-d);
      sQ[i * LK + r] = qq * ex;
    } else {
      sX[i * LK + r] = kk * gm;
    }
  }
  __syncthreads();

  // P = strict_tril(K+ K-^T), Aqk = tril(Q+ K-^T)
  if (!slow) {
    using Tl = Tiling<kC, kC>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4];
    zero(acc);
    warp_mma_kk<Tl::MT, Tl::NT, X3, DK>(acc, sX, LK, sY, LK, m0, n0);
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int j) {
      sP[i * kLC + j] = j < i ? acc[mt][nt][e] : 0.f;
    });
    zero(acc);
    warp_mma_kk<Tl::MT, Tl::NT, X3, DK>(acc, sQ, LK, sY, LK, m0, n0);
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int j) {
      sA[i * kLC + j] = j <= i ? acc[mt][nt][e] : 0.f;
    });
  } else {
    for (int idx = tid; idx < kC * kC; idx += kThreads) {
      const int i = idx / kC, j = idx % kC;
      float p = 0.f, s = 0.f;
      if (j <= i) {
        for (int r = 0; r < DK; ++r) {
          const float e = expf(sG[i * LK + r] - sG[j * LK + r]) * sK[j * LK + r];
          p = fmaf(sK[i * LK + r], e, p);
          s = fmaf(sQ[i * LK + r], e, s);
        }
      }
      sP[i * kLC + j] = j < i ? p : 0.f;
      sA[i * kLC + j] = j <= i ? a.scale * s : 0.f;
    }
  }
  __syncthreads();
  store_f32(a.Pkk + rec * kC * kC, kC, sP, kLC, kC, kC);
  for (int idx = tid; idx < kC * kC; idx += kThreads) {  // Aqk^T
    const int j = idx / kC, i = idx % kC;
    a.Aqk[rec * kC * kC + idx] = sA[i * kLC + j];
  }

  // Warps 0-7: T = (I + diag(beta) P)^-1 by 16 x 16 blocks; the other warps
  // meanwhile build beta K+ and beta v, the right operands of W and U.
  if (tid < kSolveThreads) {
    solve_T_blocked<kSolveThreads>(sP, sb, sT, sXs, tid);
  } else {
    for (int idx = tid - kSolveThreads; idx < kC * DK; idx += kThreads - kSolveThreads) {
      const int i = idx / DK, r = idx % DK;
      sX[i * LK + r] *= sb[i] * (slow ? 1.f : se[r]);
    }
    for (int idx = tid - kSolveThreads; idx < kC * DV; idx += kThreads - kSolveThreads) {
      const int i = idx / DV, c = idx % DV;
      const IO* vr = static_cast<const IO*>(a.v) + (row0 + (size_t)i * a.H) * DV;
      sY[i * LM + c] = i < nv ? sb[i] * to_f32(vr[c]) : 0.f;
    }
  }
  __syncthreads();
  store_f32(a.Tm + rec * kC * kC, kC, sT, kLC, kC, kC);
  {
    using Tl = Tiling<kC, DK>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4];
    zero(acc);
    warp_mma<Tl::MT, Tl::NT, X3, kC>(acc, rowm(sT, kLC), rowm(sX, LK), m0, n0);
    float* Wg = a.W + rec * kC * DK;
    float* Wtg = a.Wt + rec * kC * DK;
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int c) {
      Wg[i * DK + c] = acc[mt][nt][e];
      Wtg[c * kC + i] = acc[mt][nt][e];
    });
  }
  {
    using Tl = Tiling<kC, DV>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4];
    zero(acc);
    warp_mma<Tl::MT, Tl::NT, X3, kC>(acc, rowm(sT, kLC), rowm(sY, LM), m0, n0);
    float* Ug = a.U + rec * kC * DV;
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int c) { Ug[i * DV + c] = acc[mt][nt][e]; });
  }
}


// ------------------------------------------------------------------ kernel 2
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Shared-memory plan of the pass kernel (floats).  Every product operand is
// K-contiguous (ldmatrix fragments): the state columns, V', dS, dV' and dO are
// kept transposed ([column][row]) and the chunk operands come transposed from
// the prep kernel where the product needs it.  Role 0 keeps S^T and V'^T and
// NB0 buffers of {W, Kbar^T, U columns, gamma}; role 1 keeps dS^T, dV'^T,
// dO^T, Q+^T, W^T and NB1 buffers of {Aqk^T, Kbar, gamma, raw dO columns}.
// Two buffers (the next chunk's operands load while this one computes) where
// they fit.
template <int DK, int DV, int SW>
struct PassPlan {
  static constexpr int LK = DK + 4, LS = SW + 4;
  static constexpr size_t kMax = 232448 / sizeof(float);
  static constexpr size_t fix0 = (size_t)SW * LK + SW * kLC;
  static constexpr size_t buf0 = (size_t)kC * LK + (size_t)DK * kLC + kC * LS + DK;
  static constexpr size_t fix1 = (size_t)SW * LK + 2 * SW * kLC + 2 * (size_t)DK * kLC;
  static constexpr size_t stage1 = (size_t)kC * SW * 4 / sizeof(float);  // raw dO columns, up to 4 bytes each
  static constexpr size_t buf1 = (size_t)kC * kLC + (size_t)kC * LK + DK + stage1;
  static constexpr int NB0 = fix0 + 2 * buf0 <= kMax ? 2 : 1;
  static constexpr int NB1 = fix1 + 2 * buf1 <= kMax ? 2 : 1;
  static constexpr size_t r0 = fix0 + NB0 * buf0, r1 = fix1 + NB1 * buf1;
  static constexpr size_t bytes = sizeof(float) * (r0 > r1 ? r0 : r1);
};
template <int DK, int DV, int SW>
constexpr size_t pass_smem() {
  return PassPlan<DK, DV, SW>::bytes;
}

// A DK x SW block of the state (rows r, columns c) held transposed in shared
// memory (sT[c * ld + r]) to / from its place in a [DK][DV] fp32 array.
template <int NTH, int DK, int SW>
__device__ __forceinline__ void store_state_t(float* g, int DV, const float* sT, int ld) {
  for (int idx = threadIdx.x; idx < DK * (SW / 4); idx += NTH) {
    const int r = idx / (SW / 4), c = (idx % (SW / 4)) * 4;
    *reinterpret_cast<float4*>(g + (size_t)r * DV + c) =
        make_float4(sT[c * ld + r], sT[(c + 1) * ld + r], sT[(c + 2) * ld + r], sT[(c + 3) * ld + r]);
  }
}
template <int NTH, int DK, int SW>
__device__ __forceinline__ void load_state_t(float* sT, int ld, const float* g, int DV) {
  for (int idx = threadIdx.x; idx < DK * (SW / 4); idx += NTH) {
    const int r = idx / (SW / 4), c = (idx % (SW / 4)) * 4;
    const float4 x = g ? *reinterpret_cast<const float4*>(g + (size_t)r * DV + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    sT[c * ld + r] = x.x, sT[(c + 1) * ld + r] = x.y, sT[(c + 2) * ld + r] = x.z, sT[(c + 3) * ld + r] = x.w;
  }
}

// One CTA per (sequence, head, SW-column slice of the state) and role:
// role 0 replays the forward over the chunks from S_0 and stores each chunk's
// entering state and V'; role 1 walks the chunks backwards from dL/dS_T and
// stores dL/d(state leaving the chunk) and dV', and writes dL/dS_0.
template <typename IO, int DK, int DV, int SW>
__global__ void __launch_bounds__(kPassThreads, 1) bwd_pass_kernel(const ChunkBwdArgs a) {
  pdl_wait();  // the previous kernel of the call has finished
  pdl_trigger();
  constexpr bool X3 = std::is_same<IO, float>::value;
  using PP = PassPlan<DK, DV, SW>;
  constexpr int LK = PP::LK, LS = PP::LS, NS = DV / SW;
  constexpr int NTH = kPassThreads;
  using TV = Tiling<kC, SW, NTH / 32>;  // 64 x SW products
  using TS = Tiling<DK, SW, NTH / 32>;  // DK x SW products
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int cs = blockIdx.x % NS, lb = blockIdx.x / NS, bh = a.bh0 + lb, c0 = cs * SW, NC = a.NC;
  const size_t st0 = (size_t)bh * DK * DV;
  const int vm0 = TV::m0(warp), vn0 = TV::n0(warp), sm0 = TS::m0(warp), sn0 = TS::n0(warp);

  if (blockIdx.y == 0) {
    constexpr int NB = PP::NB0;
    float* sSt = sm;             // [SW][LK] state columns, transposed
    float* sVt = sSt + SW * LK;  // [SW][kLC] V', transposed
    float* sbuf = sVt + SW * kLC;
    auto sW = [&](int p) { return sbuf + p * PP::buf0; };                                   // [64][LK] W
    auto sKbt = [&](int p) { return sbuf + p * PP::buf0 + kC * LK; };                       // [DK][kLC] Kbar^T
    auto sU = [&](int p) { return sbuf + p * PP::buf0 + kC * LK + DK * kLC; };              // [64][LS] U columns
    auto sgm = [&](int p) { return sbuf + p * PP::buf0 + kC * LK + DK * kLC + kC * LS; };   // [DK] gamma
    auto issue = [&](int n, int p) {
      const size_t rec = (size_t)lb * NC + n;
      load_f32<NTH>(sW(p), LK, a.W + rec * kC * DK, DK, kC, DK);
      load_f32<NTH>(sKbt(p), kLC, a.Kbt + rec * kC * DK, kC, DK, kC);
      load_f32<NTH>(sU(p), LS, a.U + rec * kC * DV + c0, DV, kC, SW);
      load_f32<NTH>(sgm(p), DK, a.gam + rec * DK, DK, 1, DK);
      cp_commit();
    };
    load_state_t<NTH, DK, SW>(sSt, LK, a.s0 ? a.s0 + st0 + c0 : nullptr, DV);
    issue(0, 0);
    for (int n = 0; n < NC; ++n) {
      const size_t rec = (size_t)lb * NC + n;
      const int p = NB == 2 ? (n & 1) : 0;
      __syncthreads();  // the previous chunk's reads are done
      if (NB == 1 && n > 0) issue(n, 0);
      store_state_t<NTH, DK, SW>(a.S0c + rec * DK * DV + c0, DV, sSt, LK);
      cp_wait_group<0>();
      __syncthreads();
      if (NB == 2 && n + 1 < NC) issue(n + 1, p ^ 1);
      {  // V' = U - W S
        float acc[TV::MT][TV::NT][4];
        zero(acc);
        warp_mma_kk<TV::MT, TV::NT, X3, DK>(acc, sW(p), LK, sSt, LK, vm0, vn0);
        float* vp = a.Vp + rec * kC * DV + c0;
        const float* u = sU(p);
        for_acc<TV::MT, TV::NT>(vm0, vn0, [&](int mt, int nt, int e, int i, int c) {
          const float x = u[i * LS + c] - acc[mt][nt][e];
          sVt[c * kLC + i] = x;
          vp[i * DV + c] = x;
        });
      }
      __syncthreads();
      {  // S = diag(gamma) S + Kbar^T V'
        float acc[TS::MT][TS::NT][4];
        const float* gm = sgm(p);
        for_acc<TS::MT, TS::NT>(sm0, sn0, [&](int mt, int nt, int e, int r, int c) {
          acc[mt][nt][e] = gm[r] * sSt[c * LK + r];
        });
        warp_mma_kk<TS::MT, TS::NT, X3, kC>(acc, sKbt(p), kLC, sVt, kLC, sm0, sn0);
        for_acc<TS::MT, TS::NT>(sm0, sn0,
                                [&](int mt, int nt, int e, int r, int c) { sSt[c * LK + r] = acc[mt][nt][e]; });
      }
    }
  } else {
    constexpr int NB = PP::NB1;
    float* sDt = sm;                // [SW][LK] dS columns, transposed
    float* sdVt = sDt + SW * LK;    // [SW][kLC] dV', transposed
    float* sOt = sdVt + SW * kLC;   // [SW][kLC] dO columns, transposed
    float* sQpt = sOt + SW * kLC;   // [DK][kLC] Q+^T
    float* sWt = sQpt + DK * kLC;   // [DK][kLC] W^T
    float* sbuf = sWt + DK * kLC;
    auto sAt = [&](int p) { return sbuf + p * PP::buf1; };                        // [64][kLC] Aqk^T
    auto sKb = [&](int p) { return sbuf + p * PP::buf1 + kC * kLC; };             // [64][LK] Kbar
    auto sgm = [&](int p) { return sbuf + p * PP::buf1 + kC * kLC + kC * LK; };   // [DK] gamma
    auto sraw = [&](int p) {  // [64][SW] dO columns as stored (IO)
      return reinterpret_cast<IO*>(sbuf + p * PP::buf1 + kC * kLC + kC * LK + DK);
    };
    const IO* d_o = static_cast<const IO*>(a.d_o);
    auto issue = [&](int n, int p) {
      const size_t rec = (size_t)lb * NC + n;
      load_f32<NTH>(sAt(p), kLC, a.Aqk + rec * kC * kC, kC, kC, kC);
      load_f32<NTH>(sKb(p), LK, a.Kb + rec * kC * DK, DK, kC, DK);
      load_f32<NTH>(sgm(p), DK, a.gam + rec * DK, DK, 1, DK);
      constexpr int V = 16 / sizeof(IO), PER = SW / V;  // 16-byte pieces per row
      const int t0 = n * kC, nv = min(kC, a.T - t0);
      const size_t r0 = row_of(a, bh, t0);
      for (int idx = tid; idx < kC * PER; idx += NTH) {
        const int i = idx / PER, c = (idx % PER) * V;
        const IO* src = i < nv ? d_o + (r0 + (size_t)i * a.H) * DV + c0 + c : d_o;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         (uint32_t)__cvta_generic_to_shared(sraw(p) + i * SW + c)),
                     "l"(src), "r"(i < nv ? 16 : 0)
                     : "memory");
      }
      cp_commit();
    };
    load_state_t<NTH, DK, SW>(sDt, LK, a.dsT ? a.dsT + st0 + c0 : nullptr, DV);
    issue(NC - 1, NB == 2 ? ((NC - 1) & 1) : 0);
    for (int n = NC - 1; n >= 0; --n) {
      const size_t rec = (size_t)lb * NC + n;
      const int p = NB == 2 ? (n & 1) : 0;
      __syncthreads();  // the previous chunk's reads are done
      if (NB == 1 && n < NC - 1) issue(n, 0);
      store_state_t<NTH, DK, SW>(a.dSc + rec * DK * DV + c0, DV, sDt, LK);
      load_f32<NTH>(sQpt, kLC, a.Qpt + rec * kC * DK, kC, DK, kC);
      load_f32<NTH>(sWt, kLC, a.Wt + rec * kC * DK, kC, DK, kC);
      cp_commit();
      cp_wait_group<1>();  // this chunk's Aqk^T, Kbar, gamma, dO (Q+^T and W^T may still be in flight)
      __syncthreads();
      for (int idx = tid; idx < kC * SW; idx += NTH) {  // dO columns to fp32, transposed (zeros past the tail)
        const int c = idx / kC, i = idx % kC;
        sOt[c * kLC + i] = to_f32(sraw(p)[i * SW + c]);
      }
      __syncthreads();
      {  // dV' = Aqk^T dO + Kbar dS
        float acc[TV::MT][TV::NT][4];
        zero(acc);
        warp_mma_kk<TV::MT, TV::NT, X3, kC>(acc, sAt(p), kLC, sOt, kLC, vm0, vn0);
        warp_mma_kk<TV::MT, TV::NT, X3, DK>(acc, sKb(p), LK, sDt, LK, vm0, vn0);
        float* dvp = a.dVp + rec * kC * DV + c0;
        for_acc<TV::MT, TV::NT>(vm0, vn0, [&](int mt, int nt, int e, int i, int c) {
          sdVt[c * kLC + i] = acc[mt][nt][e];
          dvp[i * DV + c] = acc[mt][nt][e];
        });
      }
      if (NB == 2 && n > 0) {
        issue(n - 1, p ^ 1);
        cp_wait_group<1>();  // Q+^T and W^T of this chunk
      } else {
        cp_wait_group<0>();
      }
      __syncthreads();
      {  // dS = diag(gamma) dS + Q+^T dO - W^T dV'
        float acc[TS::MT][TS::NT][4], neg[TS::MT][TS::NT][4];
        const float* gm = sgm(p);
        for_acc<TS::MT, TS::NT>(sm0, sn0, [&](int mt, int nt, int e, int r, int c) {
          acc[mt][nt][e] = gm[r] * sDt[c * LK + r];
        });
        warp_mma_kk<TS::MT, TS::NT, X3, kC>(acc, sQpt, kLC, sOt, kLC, sm0, sn0);
        zero(neg);
        warp_mma_kk<TS::MT, TS::NT, X3, kC>(neg, sWt, kLC, sdVt, kLC, sm0, sn0);
        for_acc<TS::MT, TS::NT>(sm0, sn0, [&](int mt, int nt, int e, int r, int c) {
          sDt[c * LK + r] = acc[mt][nt][e] - neg[mt][nt][e];
        });
      }
    }
    __syncthreads();
    if (a.ds0) store_state_t<NTH, DK, SW>(a.ds0 + st0 + c0, DV, sDt, LK);
  }
}

// ------------------------------------------------------------------ kernel 2 (bf16 operands)
// With bf16 inputs the state passes run on bf16 operand images and
// mma.m16n8k16 (bf16 in, fp32 accumulation); the state itself stays in fp32
// registers for the whole chain and is rounded only as an operand image.
// The prep kernel writes each chunk's pass operands as one bf16 record in
// the shared-memory layout (rows padded by 16 bytes), so a chunk's operands
// arrive by one contiguous cp.async copy.

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4_b(uint32_t (&r)[4], const bf16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const bf16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ void ldsm_x2_b(uint32_t (&r)[2], const bf16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}
__device__ __forceinline__ void ldsm_x2_t(uint32_t (&r)[2], const bf16* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"((uint32_t)__cvta_generic_to_shared(p)));
}

// acc[MT][NT] (rows m0.., columns n0..) += A[m0.., 0:K] B[0:K, n0..], bf16
// operands in shared memory.  A is [M][lda] (AT: stored transposed, [K][lda]),
// B is [K][ldb] (BT: stored transposed, [N][ldb]).  Fragments come from
// ldmatrix, with .trans where the stored rows run along the other index.
// Row starts 16-byte aligned; row strides = 16 (mod 128) bytes avoid conflicts.
template <int MT, int NT, int K, bool AT = false, bool BT = false>
__device__ __forceinline__ void warp_mma_bf16(float (&acc)[MT][NT][4], const bf16* A, int lda, const bf16* B, int ldb,
                                              int m0, int n0) {
  const int lane = threadIdx.x & 31, mat = lane >> 3, rr = lane & 7;
  // matrices of an A x4: (m 0-7, k 0-7), (m 8-15, k 0-7), (m 0-7, k 8-15), (m 8-15, k 8-15)
  const bf16* pa = AT ? A + (rr + 8 * (mat >> 1)) * lda + m0 + 8 * (mat & 1)
                      : A + (m0 + rr + 8 * (mat & 1)) * lda + 8 * (mat >> 1);
  // matrices of a B x4: (k 0-7, n 0-7), (k 8-15, n 0-7), (k 0-7, n 8-15), (k 8-15, n 8-15)
  const bf16* pb = BT ? B + (n0 + rr + 8 * (mat >> 1)) * ldb + 8 * (mat & 1)
                      : B + (rr + 8 * (mat & 1)) * ldb + n0 + 8 * (mat >> 1);
  // odd NT: the last B tile by an x2 (lanes 0-15)
  const bf16* pb1 = BT ? B + (n0 + 8 * (NT - 1) + rr) * ldb + 8 * (mat & 1)
                       : B + (rr + 8 * (mat & 1)) * ldb + n0 + 8 * (NT - 1);
#pragma unroll
  for (int k0 = 0; k0 < K; k0 += 16) {
    uint32_t af[MT][4], bfr[NT][2];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      if constexpr (AT)
        ldsm_x4_t(af[mt], pa + k0 * lda + 16 * mt);
      else
        ldsm_x4_b(af[mt], pa + 16 * mt * lda + k0);
    }
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      uint32_t r[4];
      if constexpr (BT)
        ldsm_x4_b(r, pb + 16 * np * ldb + k0);
      else
        ldsm_x4_t(r, pb + k0 * ldb + 16 * np);
      bfr[2 * np][0] = r[0], bfr[2 * np][1] = r[1], bfr[2 * np + 1][0] = r[2], bfr[2 * np + 1][1] = r[3];
    }
    if constexpr (NT % 2 == 1) {
      uint32_t r[2];
      if constexpr (BT)
        ldsm_x2_b(r, pb1 + k0);
      else
        ldsm_x2_t(r, pb1 + k0 * ldb);
      bfr[NT - 1][0] = r[0], bfr[NT - 1][1] = r[1];
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[mt][nt], af[mt], bfr[nt][0], bfr[nt][1]);
  }
}

// The accumulator tile as a bf16 image: rows and column pairs of this lane.
template <int MT, int NT>
__device__ __forceinline__ void acc_to_bf16(const float (&acc)[MT][NT][4], bf16* img, int ld, int m0, int n0) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = m0 + 16 * mt + g + 8 * hh, c = n0 + 8 * nt + 2 * t;
        *reinterpret_cast<__nv_bfloat162*>(img + r * ld + c) =
            __floats2bfloat162_rn(acc[mt][nt][2 * hh], acc[mt][nt][2 * hh + 1]);
      }
}
// ... and as fp32 into a [rows][gld] global array (column pairs as float2).
template <int MT, int NT>
__device__ __forceinline__ void acc_to_global(const float (&acc)[MT][NT][4], float* g0, size_t gld, int m0, int n0) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = m0 + 16 * mt + g + 8 * hh, c = n0 + 8 * nt + 2 * t;
        *reinterpret_cast<float2*>(g0 + r * gld + c) = make_float2(acc[mt][nt][2 * hh], acc[mt][nt][2 * hh + 1]);
      }
}

template <int DK, int DV, int SW>
struct PassPlanB {  // bytes
  using R = PassRec<DK>;
  static constexpr int LS = SW + 8;  // bf16 images of the state / V' / dV' / dO columns
  static constexpr size_t img = (size_t)(DK + kC) * LS * 2;
  static constexpr size_t buf0 = (size_t)(R::n - R::oW) * 2 + DK * 4 + (size_t)kC * SW * 4;  // W, Kbar, gamma, U
  static constexpr size_t buf1 = (size_t)R::n * 2 + DK * 4 + (size_t)kC * LS * 2;            // record, gamma, dO
  static constexpr size_t bytes = img + 2 * (buf0 > buf1 ? buf0 : buf1);
  static_assert(img % 16 == 0 && buf0 % 16 == 0 && buf1 % 16 == 0, "16 B");
};
template <int DK, int DV, int SW>
constexpr size_t pass_bf16_smem() {
  return PassPlanB<DK, DV, SW>::bytes;
}

template <int DK, int DV, int SW>
__global__ void __launch_bounds__(kPassThreads, 1) bwd_pass_bf16_kernel(const ChunkBwdArgs a) {
  pdl_wait();  // the previous kernel of the call has finished
  pdl_trigger();
  using PB = PassPlanB<DK, DV, SW>;
  using R = PassRec<DK>;
  constexpr int LS = PB::LS, NS = DV / SW, NTH = kPassThreads;
  constexpr size_t BUF = PB::buf0 > PB::buf1 ? PB::buf0 : PB::buf1;
  using TV = Tiling<kC, SW, NTH / 32>;  // 64 x SW products
  using TS = Tiling<DK, SW, NTH / 32>;  // DK x SW products (the state, in registers)
  extern __shared__ __align__(16) uint8_t smb[];
  const int tid = threadIdx.x, warp = tid >> 5;
  const int cs = blockIdx.x % NS, lb = blockIdx.x / NS, bh = a.bh0 + lb, c0 = cs * SW, NC = a.NC;
  const size_t st0 = (size_t)bh * DK * DV;
  const int vm0 = TV::m0(warp), vn0 = TV::n0(warp), sm0 = TS::m0(warp), sn0 = TS::n0(warp);
  bf16* simg = reinterpret_cast<bf16*>(smb);      // [DK][LS] state (or dS) image
  bf16* vimg = simg + DK * LS;                    // [64][LS] V' (or dV') image
  uint8_t* bufs = smb + PB::img;
  auto copy = [&](uint8_t* dst, const void* src, size_t bytes) {  // bytes % 16 == 0
    const uint8_t* s = static_cast<const uint8_t*>(src);
    for (size_t o = (size_t)tid * 16; o < bytes; o += (size_t)NTH * 16) cp16(dst + o, s + o, 16);
  };
  float st[TS::MT][TS::NT][4];  // the state (or dS) columns of this warp's tile
  const float* init = blockIdx.y == 0 ? a.s0 : a.dsT;
  for_acc<TS::MT, TS::NT>(sm0, sn0, [&](int mt, int nt, int e, int r, int c) {
    st[mt][nt][e] = init ? init[st0 + (size_t)r * DV + c0 + c] : 0.f;
  });

  if (blockIdx.y == 0) {
    // buffer: W, Kbar [64][LKb] (bf16), gamma [DK], U columns [64][SW] (fp32)
    auto bW = [&](int p) { return reinterpret_cast<const bf16*>(bufs + p * BUF); };
    auto bKb = [&](int p) { return bW(p) + (R::oKb - R::oW); };
    auto bgm = [&](int p) { return reinterpret_cast<const float*>(bufs + p * BUF + (R::n - R::oW) * 2); };
    auto bU = [&](int p) { return bgm(p) + DK; };
    auto issue = [&](int n, int p) {
      const size_t rec = (size_t)lb * NC + n;
      uint8_t* b = bufs + p * BUF;
      copy(b, a.prec + rec * R::n + R::oW, (size_t)(R::n - R::oW) * 2);
      copy(b + (R::n - R::oW) * 2, a.gam + rec * DK, DK * 4);
      float* u = const_cast<float*>(bU(p));
      const float* ug = a.U + rec * kC * DV + c0;
      for (int idx = tid; idx < kC * (SW / 4); idx += NTH) {
        const int i = idx / (SW / 4), c = (idx % (SW / 4)) * 4;
        cp16(u + i * SW + c, ug + (size_t)i * DV + c, 16);
      }
      cp_commit();
    };
    issue(0, 0);
    for (int n = 0; n < NC; ++n) {
      const size_t rec = (size_t)lb * NC + n;
      const int p = n & 1;
      acc_to_bf16(st, simg, LS, sm0, sn0);
      acc_to_bf16(st, reinterpret_cast<bf16*>(a.S0c) + rec * DK * DV + c0, DV, sm0, sn0);
      cp_wait_group<0>();
      __syncthreads();
      if (n + 1 < NC) issue(n + 1, p ^ 1);
      {  // V' = U - W S
        float acc[TV::MT][TV::NT][4];
        zero(acc);
        warp_mma_bf16<TV::MT, TV::NT, DK>(acc, bW(p), R::LKb, simg, LS, vm0, vn0);
        const float* u = bU(p);
        for_acc<TV::MT, TV::NT>(vm0, vn0,
                                [&](int mt, int nt, int e, int i, int c) { acc[mt][nt][e] = u[i * SW + c] - acc[mt][nt][e]; });
        acc_to_bf16(acc, vimg, LS, vm0, vn0);
        acc_to_bf16(acc, reinterpret_cast<bf16*>(a.Vp) + rec * kC * DV + c0, DV, vm0, vn0);
      }
      __syncthreads();
      {  // S = diag(gamma) S + Kbar^T V'
        const float* gm = bgm(p);
        for_acc<TS::MT, TS::NT>(sm0, sn0, [&](int mt, int nt, int e, int r, int c) { st[mt][nt][e] *= gm[r]; });
        warp_mma_bf16<TS::MT, TS::NT, kC, true>(st, bKb(p), R::LKb, vimg, LS, sm0, sn0);
      }
    }
  } else {
    // buffer: the record (Aqk, Q+, W, Kbar; bf16), gamma [DK], dO columns [64][LS] (bf16)
    auto bR = [&](int p) { return reinterpret_cast<const bf16*>(bufs + p * BUF); };
    auto bgm = [&](int p) { return reinterpret_cast<const float*>(bufs + p * BUF + R::n * 2); };
    auto bO = [&](int p) { return reinterpret_cast<const bf16*>(bufs + p * BUF + R::n * 2 + DK * 4); };
    const bf16* d_o = static_cast<const bf16*>(a.d_o);
    auto issue = [&](int n, int p) {
      const size_t rec = (size_t)lb * NC + n;
      uint8_t* b = bufs + p * BUF;
      copy(b, a.prec + rec * R::n, (size_t)R::n * 2);
      copy(b + R::n * 2, a.gam + rec * DK, DK * 4);
      constexpr int PER = SW / 8;  // 16-byte pieces per row
      const int t0 = n * kC, nv = min(kC, a.T - t0);
      const size_t r0 = row_of(a, bh, t0);
      bf16* o = const_cast<bf16*>(bO(p));
      for (int idx = tid; idx < kC * PER; idx += NTH) {
        const int i = idx / PER, c = (idx % PER) * 8;
        cp16(o + i * LS + c, i < nv ? d_o + (r0 + (size_t)i * a.H) * DV + c0 + c : d_o, i < nv ? 16 : 0);
      }
      cp_commit();
    };
    issue(NC - 1, (NC - 1) & 1);
    for (int n = NC - 1; n >= 0; --n) {
      const size_t rec = (size_t)lb * NC + n;
      const int p = n & 1;
      acc_to_bf16(st, simg, LS, sm0, sn0);
      acc_to_bf16(st, reinterpret_cast<bf16*>(a.dSc) + rec * DK * DV + c0, DV, sm0, sn0);
      cp_wait_group<0>();
      __syncthreads();
      if (n > 0) issue(n - 1, p ^ 1);
      const bf16* rp = bR(p);
      {  // dV' = Aqk^T dO + Kbar dS
        float acc[TV::MT][TV::NT][4];
        zero(acc);
        warp_mma_bf16<TV::MT, TV::NT, kC, true>(acc, rp + R::oAqk, R::LCb, bO(p), LS, vm0, vn0);
        warp_mma_bf16<TV::MT, TV::NT, DK>(acc, rp + R::oKb, R::LKb, simg, LS, vm0, vn0);
        acc_to_bf16(acc, vimg, LS, vm0, vn0);
        acc_to_bf16(acc, reinterpret_cast<bf16*>(a.dVp) + rec * kC * DV + c0, DV, vm0, vn0);
      }
      __syncthreads();
      {  // dS = diag(gamma) dS + Q+^T dO - W^T dV'
        const float* gm = bgm(p);
        float neg[TS::MT][TS::NT][4];
        for_acc<TS::MT, TS::NT>(sm0, sn0, [&](int mt, int nt, int e, int r, int c) { st[mt][nt][e] *= gm[r]; });
        warp_mma_bf16<TS::MT, TS::NT, kC, true>(st, rp + R::oQp, R::LKb, bO(p), LS, sm0, sn0);
        zero(neg);
        warp_mma_bf16<TS::MT, TS::NT, kC, true>(neg, rp + R::oW, R::LKb, vimg, LS, sm0, sn0);
        for_acc<TS::MT, TS::NT>(sm0, sn0, [&](int mt, int nt, int e, int r, int c) { st[mt][nt][e] -= neg[mt][nt][e]; });
      }
    }
    if (a.ds0)
      for_acc<TS::MT, TS::NT>(sm0, sn0, [&](int mt, int nt, int e, int r, int c) {
        a.ds0[st0 + (size_t)r * DV + c0 + c] = st[mt][nt][e];
      });
  }
}

// ------------------------------------------------------------------ kernel 2, tensor-core form
// The two state passes for bf16 inputs at d_k = d_v = 128 on the tcgen05
// tensor cores, one CTA per (sequence, head) and role, with the state kept
// transposed in tensor memory (lane j = value channel j, 128 fp32 columns =
// key channels) for the whole chain, as in the forward's state pass:
//   role 0 (replay, chunks in order):   P = S0^T W^T;  V'^T = U^T - P;
//                                       S^T <- S^T diag(gamma) + V'^T Kbar
//   role 1 (reverse sweep, backwards):  dV'^T = dO^T Aqk + dS^T Kbar^T;
//                                       dS^T <- dS^T diag(gamma) + dO^T Q+ - dV'^T W
// Every product has M = 128 (the value channels): A is the state (or V'^T,
// dV'^T) in bf16 from tensor memory, or dO^T read MN-major from the TMA
// tile of dO; B is a token-row tile of the record (W, Kbar as K-major or
// MN-major views, Q+, Aqk).  Warps 0-3 own the state rows: they convert the
// state and V' to bf16 operands, decay the state by gamma, form V'^T = U^T - P,
// and write the bf16 checkpoints (S0 or dS entering the chunk's step, V' or
// dV') in the row-major layouts the per-chunk kernels read.  Warp 4 issues
// the MMAs, warp 5 streams each chunk's operands into one of two stages.
// Every mbarrier wait is bounded; a give-up sets the workspace error word.
namespace tcpass {
using namespace sm100;
constexpr int kThreads = 192;
constexpr uint32_t kStage = 83968;                                   // bytes per stage (82 KiB)
constexpr uint32_t kStW = 0, kStQ = 16384, kStKb = 32768, kStAqk = 49152;  // record tiles (as in TcRec)
constexpr uint32_t kStO = 57344;   // role 1: the dO tile, [64 tokens][2 x 64 value channels]
constexpr uint32_t kStU = 49152;   // role 0: U (fp32 [64][128])
constexpr uint32_t kStGam = 81920; // gamma (fp32 [128])
constexpr size_t kSmem = 2 * (size_t)kStage + 1024;
constexpr uint32_t kTmAcc = 0, kTmS = 64, kTmAS = 192, kTmAV = 256;  // tensor-memory columns
constexpr uint32_t kWait = 1u << 24;
static_assert(kStU + 32768 <= kStGam && kStO + 16384 <= kStGam && kStGam + 512 <= kStage, "stage layout");

__device__ __forceinline__ void wait_or_flag(uint64_t* bar, uint32_t parity, WorkspaceHeader* hdr, uint32_t where) {
  if (!mbar_wait(bar, parity, kWait)) {
    atomicOr(&hdr->error, 1u);
    atomicExch(&hdr->where, where);
  }
}
__device__ __forceinline__ uint32_t pk2(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}

__global__ void __launch_bounds__(kThreads, 1)
    bwd_pass_tc_kernel(const __grid_constant__ CUtensorMap tm_do, const ChunkBwdArgs a, WorkspaceHeader* hdr) {
  constexpr int DK = 128, DV = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_full[2], bar_free[2], bar_as, bar_p, bar_av, bar_s;
  __shared__ uint32_t tmem_base;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int role = blockIdx.y, lb = blockIdx.x, bh = a.bh0 + lb, NC = a.NC;
  const int h = bh % a.H, b = bh / a.H;
  const size_t st0 = (size_t)bh * DK * DV;
  const uint8_t* recs = reinterpret_cast<const uint8_t*>(a.prec) + (size_t)lb * NC * (PassRec<DK>::n * 2);
  if (tid == 0) prefetch_tensormap(&tm_do);
  pdl_wait();  // the preparation kernel has finished
  pdl_trigger();
  if (tid == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(&bar_free[0], 1);
    mbar_init(&bar_free[1], 1);
    mbar_init(&bar_as, 128);
    mbar_init(&bar_p, 1);
    mbar_init(&bar_av, 128);
    mbar_init(&bar_s, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_base;
  auto chunk_of = [&](int it) { return role ? NC - 1 - it : it; };

  if (warp == 5) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      auto load = [&](int it) {
        const int n = chunk_of(it), s = it & 1;
        uint8_t* st = sm + s * kStage;
        const size_t rec = (size_t)lb * NC + n;
        const uint8_t* rp = recs + (size_t)n * (PassRec<DK>::n * 2);
        if (role == 0) {
          mbar_expect_tx(&bar_full[s], 2 * 16384 + 32768 + 512);
          bulk_load(st + kStW, rp + TcRec::oW, 16384, &bar_full[s]);
          bulk_load(st + kStKb, rp + TcRec::oKb, 16384, &bar_full[s]);
          bulk_load(st + kStU, a.U + rec * kC * DV, 32768, &bar_full[s]);
        } else {
          mbar_expect_tx(&bar_full[s], TcRec::bytes + 16384 + 512);
          bulk_load(st, rp, TcRec::bytes, &bar_full[s]);
          tma_load_4d(st + kStO, &tm_do, &bar_full[s], 0, h, n * kC, b);
          tma_load_4d(st + kStO + 8192, &tm_do, &bar_full[s], 64, h, n * kC, b);
        }
        bulk_load(st + kStGam, a.gam + rec * DK, 512, &bar_full[s]);
      };
      for (int it = 0; it < 2 && it < NC; ++it) load(it);
      // A stage is refilled once the products of the chunk it held are done
      // (every read of it by the state rows precedes their last arrival).
      for (int it = 0; it + 2 < NC; ++it) {
        wait_or_flag(&bar_free[it & 1], (it >> 1) & 1, hdr, 60);
        load(it + 2);
      }
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t id_k64 = idesc_bf16_f32(128, 64, 0, 0);    // A tensor memory, B K-major, N = 64 tokens
      const uint32_t id_m128 = idesc_bf16_f32(128, 128, 0, 1);  // A tensor memory, B MN-major, N = 128 channels
      const uint32_t id_o64 = idesc_bf16_f32(128, 64, 1, 1);    // A = dO^T (MN-major), B MN-major, N = 64
      const uint32_t id_o128 = idesc_bf16_f32(128, 128, 1, 1);  // A = dO^T, B MN-major, N = 128
      for (int it = 0; it < NC; ++it) {
        const int s = it & 1;
        const uint32_t st = smem_u32(sm + s * kStage);
        wait_or_flag(&bar_full[s], (it >> 1) & 1, hdr, 61);
        wait_or_flag(&bar_as, it & 1, hdr, 62);
        tc_fence_after();
        // K-major view of a token-row tile: 16 channels per step, +8 KiB per 64-channel block
        auto kview = [&](uint32_t off, int k) {
          return desc_sw128(st + off, 16, 1024) + (uint64_t)((((k >> 2) * 8192) + (k & 3) * 32) >> 4);
        };
        // MN-major view (N or M = channels, two 64-wide blocks 8 KiB apart): 16 tokens per step
        auto mview = [&](uint32_t off, int k) { return desc_sw128(st + off, 8192, 1024) + (uint64_t)((2 * k * 1024) >> 4); };
        if (role == 0) {
#pragma unroll
          for (int k = 0; k < DK / 16; ++k)  // P = S0^T W^T
            mma_bf16_ts(tm + kTmAcc, tm + kTmAS + k * 8, kview(kStW, k), id_k64, k > 0);
        } else {
#pragma unroll
          for (int k = 0; k < kC / 16; ++k)  // dV'^T = dO^T Aqk ...
            mma_bf16(tm + kTmAcc, mview(kStO, k), mview(kStAqk, k), id_o64, k > 0);
#pragma unroll
          for (int k = 0; k < DK / 16; ++k)  // ... + dS^T Kbar^T
            mma_bf16_ts(tm + kTmAcc, tm + kTmAS + k * 8, kview(kStKb, k), id_k64, 1);
        }
        mma_commit(&bar_p);
        wait_or_flag(&bar_av, it & 1, hdr, 63);
        tc_fence_after();
        if (role == 0) {
#pragma unroll
          for (int k = 0; k < kC / 16; ++k)  // S^T += V'^T Kbar
            mma_bf16_ts(tm + kTmS, tm + kTmAV + k * 8, mview(kStKb, k), id_m128, 1);
        } else {
#pragma unroll
          for (int k = 0; k < kC / 16; ++k)  // dS^T += dO^T Q+ ...
            mma_bf16(tm + kTmS, mview(kStO, k), mview(kStQ, k), id_o128, 1);
#pragma unroll
          for (int k = 0; k < kC / 16; ++k)  // ... + (-dV'^T) W
            mma_bf16_ts(tm + kTmS, tm + kTmAV + k * 8, mview(kStW, k), id_m128, 1);
        }
        mma_commit(&bar_s);
        mma_commit(&bar_free[s]);
      }
    }
  } else {
    // ------------------------------------------------------------ state rows
    const int j = tid;  // value channel = tensor-memory lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    {
      const float* init = role == 0 ? a.s0 : a.dsT;
#pragma unroll
      for (int q = 0; q < DK / 32; ++q) {
        float v[32];
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) v[ii] = init ? init[st0 + (size_t)(q * 32 + ii) * DV + j] : 0.f;
        tmem_st32(tm + kTmS + lane_off + q * 32, v);
      }
      tmem_wait_st();
    }
    bf16* ck_state = reinterpret_cast<bf16*>(role == 0 ? a.S0c : a.dSc);
    bf16* ck_v = reinterpret_cast<bf16*>(role == 0 ? a.Vp : a.dVp);
    // The checkpoints are written after the arrivals the MMA warp waits for,
    // so that their stores stay off the chain's critical path.
    for (int it = 0; it < NC; ++it) {
      const int n = chunk_of(it), s = it & 1;
      const size_t rec = (size_t)lb * NC + n;
      const uint8_t* st = sm + s * kStage;
      if (it > 0) wait_or_flag(&bar_s, (it - 1) & 1, hdr, 64);
      tc_fence_after();
      // (1) the state as a bf16 operand (the MMA warp waits for it)
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t r[64];
        tmem_ld32_raw(tm + kTmS + lane_off + half * 64, r);
        tmem_ld32_raw(tm + kTmS + lane_off + half * 64 + 32, r + 32);
        tmem_wait_ld();
        reg_pin<64>(r);
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pk2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
        tmem_st32u(tm + kTmAS + lane_off + half * 32, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_as);
      // (2) the state times diag(gamma), while the first products run
      wait_or_flag(&bar_full[s], (it >> 1) & 1, hdr, 65);
      {
        const float4* gam = reinterpret_cast<const float4*>(st + kStGam);
#pragma unroll
        for (int cb = 0; cb < DK / 32; ++cb) {
          uint32_t r[32];
          tmem_ld32_raw(tm + kTmS + lane_off + cb * 32, r);
          tmem_wait_ld();
          reg_pin<32>(r);
          float v[32];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 gg = gam[cb * 8 + q4];
            v[q4 * 4 + 0] = __uint_as_float(r[q4 * 4 + 0]) * gg.x;
            v[q4 * 4 + 1] = __uint_as_float(r[q4 * 4 + 1]) * gg.y;
            v[q4 * 4 + 2] = __uint_as_float(r[q4 * 4 + 2]) * gg.z;
            v[q4 * 4 + 3] = __uint_as_float(r[q4 * 4 + 3]) * gg.w;
          }
          tmem_st32(tm + kTmS + lane_off + cb * 32, v);
        }
      }
      // (3) checkpoint of the state (S0 entering the chunk, or dS leaving it), [DK][DV] bf16,
      // from its bf16 operand image, still while the first products run
      {
        bf16* cs = ck_state + rec * DK * DV + j;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
          tmem_ld32_raw(tm + kTmAS + lane_off + half * 32, pk);
          tmem_wait_ld();
          reg_pin<32>(pk);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const __nv_bfloat162 two = *reinterpret_cast<const __nv_bfloat162*>(&pk[e]);
            cs[(size_t)(half * 64 + 2 * e) * DV] = two.x;
            cs[(size_t)(half * 64 + 2 * e + 1) * DV] = two.y;
          }
        }
      }
      // (4) V'^T = U^T - P (replay) or dV'^T (reverse sweep) as the operand (-dV'^T for the sweep)
      wait_or_flag(&bar_p, it & 1, hdr, 66);
      tc_fence_after();
      const float* u = reinterpret_cast<const float*>(st + kStU) + j;
      uint32_t vk[32];  // V' (or dV') packed, for the checkpoint
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t r[32];
        tmem_ld32_raw(tm + kTmAcc + lane_off + half * 32, r);
        tmem_wait_ld();
        reg_pin<32>(r);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int t = half * 32 + 2 * e;
          float x0 = __uint_as_float(r[2 * e]), x1 = __uint_as_float(r[2 * e + 1]);
          if (role == 0) {
            x0 = u[t * DV] - x0;
            x1 = u[(t + 1) * DV] - x1;
          }
          vk[half * 16 + e] = pk2(x0, x1);
          pk[e] = role == 0 ? vk[half * 16 + e] : (vk[half * 16 + e] ^ 0x80008000u);  // the sweep subtracts dV'^T W
        }
        tmem_st16u(tm + kTmAV + lane_off + half * 16, pk);
      }
      tmem_wait_st();  // also covers the decayed state
      tc_fence_before();
      mbar_arrive(&bar_av);
      // (5) checkpoint of V' (or dV'), [64][DV] bf16, while the second products run
      {
        bf16* cv = ck_v + rec * kC * DV + j;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const __nv_bfloat162 two = *reinterpret_cast<const __nv_bfloat162*>(&vk[e]);
          cv[(size_t)(2 * e) * DV] = two.x;
          cv[(size_t)(2 * e + 1) * DV] = two.y;
        }
      }
    }
    wait_or_flag(&bar_s, (NC - 1) & 1, hdr, 67);
    tc_fence_after();
    if (role == 1 && a.ds0) {
#pragma unroll
      for (int q = 0; q < DK / 32; ++q) {
        float v[32];
        tmem_ld32(tm + kTmS + lane_off + q * 32, v);
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) a.ds0[st0 + (size_t)(q * 32 + ii) * DV + j] = v[ii];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 512);
}
}  // namespace tcpass

// ------------------------------------------------------------------ kernel 3
template <int DK, int DV>
constexpr size_t local_a_smem() {
  constexpr int LV = DV + 4;
  return sizeof(float) * ((size_t)4 * kC * LV + kC * kLC + 2 * 32 * LV + kC + 4 * kC);
}

// Per chunk: the products that contract over the value channels.
template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1) bwd_local_a_kernel(const ChunkBwdArgs a) {
  pdl_wait();  // the previous kernel of the call has finished
  pdl_trigger();
  constexpr bool X3 = std::is_same<IO, float>::value;
  constexpr int LV = DV + 4;
  extern __shared__ __align__(16) float sm[];
  float* sO = sm;              // [64][LV] dO
  float* sVp = sO + kC * LV;   // [64][LV] V'
  float* sdV = sVp + kC * LV;  // [64][LV] dV'
  float* sv = sdV + kC * LV;   // [64][LV] v
  float* sT = sv + kC * LV;    // [64][kLC] T
  float* sS0 = sT + kC * kLC;  // [32][LV] rows of S0
  float* sdS = sS0 + 32 * LV;  // [32][LV] rows of dS
  float* sb = sdS + 32 * LV;   // [64] beta
  float* red = sb + kC;        // [4][64] row sums per column group
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % a.NC, lb = blockIdx.x / a.NC, bh = a.bh0 + lb, t0 = n * kC, nv = min(kC, a.T - t0);
  const size_t row0 = row_of(a, bh, t0), rec = (size_t)lb * a.NC + n;

  load_rows<IO, DV>(sO, LV, static_cast<const IO*>(a.d_o), row0, a.H, nv, DV, 0);
  load_rows<IO, DV>(sv, LV, static_cast<const IO*>(a.v), row0, a.H, nv, DV, 0);
  load_f32(sVp, LV, a.Vp + rec * kC * DV, DV, kC, DV);
  load_f32(sdV, LV, a.dVp + rec * kC * DV, DV, kC, DV);
  load_f32(sT, kLC, a.Tm + rec * kC * kC, kC, kC, kC);
  if (tid < kC) sb[tid] = tid < nv ? to_f32(static_cast<const IO*>(a.beta)[row0 + (size_t)tid * a.H]) : 0.f;
  cp_wait();
  __syncthreads();
  {
    using Tl = Tiling<kC, kC>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4];
    zero(acc);  // dAqk = tril(dO V'^T)
    warp_mma_kk<Tl::MT, Tl::NT, X3, DV>(acc, sO, LV, sVp, LV, m0, n0);
    float* out = a.dAqk + rec * kC * kC;
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int j) {
      out[i * kC + j] = j <= i ? acc[mt][nt][e] : 0.f;
    });
    zero(acc);  // dU (beta V)^T, strictly lower part
    warp_mma_kk<Tl::MT, Tl::NT, X3, DV>(acc, sdV, LV, sv, LV, m0, n0);
    out = a.dT1 + rec * kC * kC;
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int j) {
      out[i * kC + j] = j < i ? acc[mt][nt][e] * sb[j] : 0.f;
    });
  }
  {  // X = T^T dU: dv = beta X, dbeta part = rowsum(V . X)
    using Tl = Tiling<kC, DV>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4], rp[Tl::MT][2] = {};
    zero(acc);
    warp_mma<Tl::MT, Tl::NT, X3, kC>(acc, colm(sT, kLC), rowm(sdV, LV), m0, n0);
    IO* dv = static_cast<IO*>(a.dv);
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int c) {
      const float x = acc[mt][nt][e];
      if (i < nv) dv[(row0 + (size_t)i * a.H) * DV + c] = from_f32<IO>(sb[i] * x);
      rp[mt][e >> 1] = fmaf(x, sv[i * LV + c], rp[mt][e >> 1]);
    });
    row_sums_out<Tl::MT>(rp, m0, red + (warp / Tl::WM) * kC);
  }
  __syncthreads();
  if (tid < kC) {
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < Tiling<kC, DV>::WN; ++w) x += red[w * kC + tid];
    a.dbu[rec * kC + tid] = x;
  }

  // blocks of 32 key rows of S0 and dS: dO S0^T, -dV' S0^T, V' dS^T, rowsum(dS . S0)
  using Tr = Tiling<kC, 32>;
  const int m0 = Tr::m0(warp), n0 = Tr::n0(warp);
  for (int rb = 0; rb < DK / 32; ++rb) {
    __syncthreads();
    load_f32(sS0, LV, a.S0c + rec * DK * DV + (size_t)rb * 32 * DV, DV, 32, DV);
    load_f32(sdS, LV, a.dSc + rec * DK * DV + (size_t)rb * 32 * DV, DV, 32, DV);
    cp_wait();
    __syncthreads();
    float acc[Tr::MT][Tr::NT][4];
    zero(acc);
    warp_mma_kk<Tr::MT, Tr::NT, X3, DV>(acc, sO, LV, sS0, LV, m0, n0);
    float* out = a.dQs + rec * kC * DK + rb * 32;
    for_acc<Tr::MT, Tr::NT>(m0, n0, [&](int mt, int nt, int e, int i, int c) { out[i * DK + c] = acc[mt][nt][e]; });
    zero(acc);
    warp_mma_kk<Tr::MT, Tr::NT, X3, DV>(acc, sdV, LV, sS0, LV, m0, n0);
    out = a.dW + rec * kC * DK + rb * 32;
    for_acc<Tr::MT, Tr::NT>(m0, n0, [&](int mt, int nt, int e, int i, int c) { out[i * DK + c] = -acc[mt][nt][e]; });
    zero(acc);
    warp_mma_kk<Tr::MT, Tr::NT, X3, DV>(acc, sVp, LV, sdS, LV, m0, n0);
    out = a.dKb + rec * kC * DK + rb * 32;
    for_acc<Tr::MT, Tr::NT>(m0, n0, [&](int mt, int nt, int e, int i, int c) { out[i * DK + c] = acc[mt][nt][e]; });
#pragma unroll
    for (int rr = 0; rr < 32 / kWarps; ++rr) {  // each warp: 32 / kWarps rows of the block
      const int r = (32 / kWarps) * warp + rr;
      float x = 0.f;
      for (int c = lane; c < DV; c += 32) x = fmaf(sdS[r * LV + c], sS0[r * LV + c], x);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
      if (lane == 0) a.dgam[rec * DK + rb * 32 + r] = x;
    }
  }
}


// ------------------------------------------------------------------ kernel 1 (bf16 operands)
template <int DK, int DV>
struct PrepPlanB {  // bytes
  static constexpr int LK = DK + 4, LKb = DK + 8, LVb = DV + 8, LMb = (DK > DV ? DK : DV) + 8, LCb = kC + 8;
  static constexpr size_t oG = 0, ok = oG + (size_t)kC * LK * 4, oq = ok + (size_t)kC * LKb * 2,
                          ov = oq + (size_t)kC * LKb * 2, oX = ov + (size_t)kC * LVb * 2,
                          oY = oX + (size_t)kC * LKb * 2, oQ = oY + (size_t)kC * LMb * 2,
                          oP = oQ + (size_t)kC * LKb * 2, oT = oP + (size_t)kC * kLC * 4,
                          oTf = oT + (size_t)kC * LCb * 2, oXs = oTf + (size_t)kC * kLC * 4,
                          ob = oXs + 3 * 256 * 4, oe = ob + kC * 4, bytes = oe + DK * 4;
  static_assert(ok % 16 == 0 && oq % 16 == 0 && ov % 16 == 0 && oX % 16 == 0 && oY % 16 == 0 && oQ % 16 == 0 &&
                    oP % 16 == 0 && oT % 16 == 0 && oTf % 16 == 0 && oXs % 16 == 0 && ob % 16 == 0,
                "16 B");
};

// Per chunk, bf16 inputs (exponentials by the fast intrinsic: every exponent
// here is bounded by the factored form's span or is <= 0, and the results
// feed bf16 operands): G (fp32), the factored operands as bf16 images, P
// (fp32, for the solve) and Aqk, T by forward substitution in fp32, W and U;
// the state passes' operands go out as the chunk's bf16 pass record, T as bf16.
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1) bwd_prep_bf16_kernel(const ChunkBwdArgs a) {
  pdl_trigger();
  using PL = PrepPlanB<DK, DV>;
  using PR = PassRec<DK>;
  constexpr int LK = PL::LK, LKb = PL::LKb, LVb = PL::LVb, LMb = PL::LMb, LCb = PL::LCb;
  extern __shared__ __align__(16) uint8_t smb[];
  float* sG = reinterpret_cast<float*>(smb + PL::oG);  // [64][LK] cumulative log-gates
  bf16* sk = reinterpret_cast<bf16*>(smb + PL::ok);    // [64][LKb] k (input)
  bf16* sq = reinterpret_cast<bf16*>(smb + PL::oq);    // [64][LKb] q (input)
  bf16* sv = reinterpret_cast<bf16*>(smb + PL::ov);    // [64][LVb] v (input)
  bf16* sX = reinterpret_cast<bf16*>(smb + PL::oX);    // [64][LKb] K+_r, then beta K+
  bf16* sY = reinterpret_cast<bf16*>(smb + PL::oY);    // [64][LMb] K-_r, then beta v
  bf16* sQ = reinterpret_cast<bf16*>(smb + PL::oQ);    // [64][LKb] Q+_r
  float* sP = reinterpret_cast<float*>(smb + PL::oP);  // [64][kLC] P
  bf16* sT = reinterpret_cast<bf16*>(smb + PL::oT);    // [64][LCb] T
  float* sTf = reinterpret_cast<float*>(smb + PL::oTf);  // [64][kLC] T (fp32)
  float* sXs = reinterpret_cast<float*>(smb + PL::oXs);  // [3][16][16] solve scratch
  float* sb = reinterpret_cast<float*>(smb + PL::ob);  // [64] beta
  float* se = reinterpret_cast<float*>(smb + PL::oe);  // [DK] exp(G_ref)
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n = blockIdx.x % a.NC, lb = blockIdx.x / a.NC, bh = a.bh0 + lb, t0 = n * kC, nv = min(kC, a.T - t0);
  const size_t row0 = row_of(a, bh, t0), rec = (size_t)lb * a.NC + n;
  bf16* pr = a.prec + rec * PR::n;
  uint8_t* prb = reinterpret_cast<uint8_t*>(pr);
  const bool tcr = kTcPass<DK, DV> && a.tc_rec;  // record layout of the pass kernel that will read it
  auto aqk_at = [&](int i, int j) -> bf16* {
    return tcr ? reinterpret_cast<bf16*>(prb + TcRec::oAqk + tile_off(i, j)) : pr + PR::oAqk + i * PR::LCb + j;
  };
  auto rows_in = [&](bf16* dst, int ld, const bf16* src, int D) {  // 64 input rows of D (zeros past the tail)
    const int per = D / 8;
    for (int idx = tid; idx < kC * per; idx += kThreads) {
      const int i = idx / per, c = (idx % per) * 8;
      cp16(dst + i * ld + c, i < nv ? src + (row0 + (size_t)i * a.H) * D + c : src, i < nv ? 16 : 0);
    }
  };
  rows_in(sk, LKb, static_cast<const bf16*>(a.k), DK);
  rows_in(sq, LKb, static_cast<const bf16*>(a.q), DK);
  rows_in(sv, LVb, static_cast<const bf16*>(a.v), DV);
  if (tid < kC) sb[tid] = tid < nv ? to_f32(static_cast<const bf16*>(a.beta)[row0 + (size_t)tid * a.H]) : 0.f;
  const bool slow = load_gates_cumsum<bf16, DK>(sG, LK, static_cast<const bf16*>(a.g), a.gate, row0, a.H, nv);
  if (tid < DK) {
    se[tid] = __expf(sG[kRef * LK + tid]);
    a.gam[rec * DK + tid] = __expf(sG[(kC - 1) * LK + tid]);
  }
  cp_wait();
  __syncthreads();
  for (int idx = tid; idx < kC * DK / 2; idx += kThreads) {  // Q+, Kbar (record) and the factored operands
    const int i = idx / (DK / 2), r = (idx % (DK / 2)) * 2;     // two channels per thread
    const float2 G = *reinterpret_cast<const float2*>(sG + i * LK + r);
    const float2 GC = *reinterpret_cast<const float2*>(sG + (kC - 1) * LK + r);
    const float2 kk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sk + i * LKb + r));
    float2 qq = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sq + i * LKb + r));
    qq.x *= a.scale, qq.y *= a.scale;
    __nv_bfloat162* kb_dst = tcr
                                 ? reinterpret_cast<__nv_bfloat162*>(prb + TcRec::oKb + tile_off(i, r))
                                 : reinterpret_cast<__nv_bfloat162*>(pr + PR::oKb + i * PR::LKb + r);
    __nv_bfloat162* qp_dst = tcr
                                 ? reinterpret_cast<__nv_bfloat162*>(prb + TcRec::oQp + tile_off(i, r))
                                 : reinterpret_cast<__nv_bfloat162*>(pr + PR::oQp + i * PR::LKb + r);
    *kb_dst = __floats2bfloat162_rn(kk.x * __expf(GC.x - G.x), kk.y * __expf(GC.y - G.y));
    *qp_dst = __floats2bfloat162_rn(qq.x * __expf(G.x), qq.y * __expf(G.y));
    if (!slow) {
      const float2 Gr = *reinterpret_cast<const float2*>(sG + kRef * LK + r);
      const float dx = G.x - Gr.x, dy = G.y - Gr.y, ex = __expf(dx), ey = __expf(dy);
      *reinterpret_cast<__nv_bfloat162*>(sX + i * LKb + r) = __floats2bfloat162_rn(kk.x * ex, kk.y * ey);
      *reinterpret_cast<__nv_bfloat162*>(sY + i * LMb + r) =
          __floats2bfloat162_rn(kk.x * __expf(-dx), kk.y * __expf(-dy));
      *reinterpret_cast<__nv_bfloat162*>(sQ + i * LKb + r) = __floats2bfloat162_rn(qq.x * ex, qq.y * ey);
    }
  }
  __syncthreads();

  // P = strict_tril(K+ K-^T) (fp32, shared), Aqk = tril(Q+ K-^T) (record, transposed)
  if (!slow) {
    using Tl = Tiling<kC, kC>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4];
    zero(acc);
    warp_mma_bf16<Tl::MT, Tl::NT, DK, false, true>(acc, sX, LKb, sY, LMb, m0, n0);
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int j) {
      sP[i * kLC + j] = j < i ? acc[mt][nt][e] : 0.f;
    });
    zero(acc);
    warp_mma_bf16<Tl::MT, Tl::NT, DK, false, true>(acc, sQ, LKb, sY, LMb, m0, n0);
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int j) {
      *aqk_at(i, j) = __float2bfloat16_rn(j <= i ? acc[mt][nt][e] : 0.f);
    });
  } else {
    for (int idx = tid; idx < kC * kC; idx += kThreads) {
      const int i = idx / kC, j = idx % kC;
      float p = 0.f, s = 0.f;
      if (j <= i) {
        for (int r = 0; r < DK; ++r) {
          const float e = __expf(sG[i * LK + r] - sG[j * LK + r]) * __bfloat162float(sk[j * LKb + r]);
          p = fmaf(__bfloat162float(sk[i * LKb + r]), e, p);
          s = fmaf(__bfloat162float(sq[i * LKb + r]), e, s);
        }
      }
      sP[i * kLC + j] = j < i ? p : 0.f;
      *aqk_at(i, j) = __float2bfloat16_rn(j <= i ? a.scale * s : 0.f);
    }
  }
  __syncthreads();

  // Warps 0-7: T = (I + diag(beta) P)^-1 by blocks (fp32), then its bf16 image
  // and the global copy.  The other warps meanwhile store P and the right
  // operands beta K+ and beta v of W and U (the factored tiles are dead).
  bf16* Tg = reinterpret_cast<bf16*>(a.Tm) + rec * kC * kC;
  if (tid < kSolveThreads) {
    solve_T_blocked<kSolveThreads>(sP, sb, sTf, sXs, tid);
    for (int idx = tid; idx < kC * kC / 2; idx += kSolveThreads) {
      const int i = idx / (kC / 2), j = (idx % (kC / 2)) * 2;
      const __nv_bfloat162 t2 = __floats2bfloat162_rn(sTf[i * kLC + j], sTf[i * kLC + j + 1]);
      *reinterpret_cast<__nv_bfloat162*>(sT + i * LCb + j) = t2;
      *reinterpret_cast<__nv_bfloat162*>(Tg + i * kC + j) = t2;
    }
  } else {
    const int t2 = tid - kSolveThreads, n2 = kThreads - kSolveThreads;
    float* Pg = a.Pkk + rec * kC * kC;
    for (int idx = t2; idx < kC * kC / 4; idx += n2) {
      const int i = idx / (kC / 4), j = (idx % (kC / 4)) * 4;
      *reinterpret_cast<float4*>(Pg + i * kC + j) = *reinterpret_cast<const float4*>(sP + i * kLC + j);
    }
    for (int idx = t2; idx < kC * DK / 2; idx += n2) {
      const int i = idx / (DK / 2), r = (idx % (DK / 2)) * 2;
      const float2 kk = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sk + i * LKb + r));
      const float2 G = *reinterpret_cast<const float2*>(sG + i * LK + r);
      *reinterpret_cast<__nv_bfloat162*>(sX + i * LKb + r) =
          __floats2bfloat162_rn(sb[i] * kk.x * __expf(G.x), sb[i] * kk.y * __expf(G.y));
    }
    for (int idx = t2; idx < kC * DV / 2; idx += n2) {
      const int i = idx / (DV / 2), c = (idx % (DV / 2)) * 2;
      const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sv + i * LVb + c));
      *reinterpret_cast<__nv_bfloat162*>(sY + i * LMb + c) = __floats2bfloat162_rn(sb[i] * v.x, sb[i] * v.y);
    }
  }
  __syncthreads();
  {  // W = T (beta K+): record
    using Tl = Tiling<kC, DK>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4];
    zero(acc);
    warp_mma_bf16<Tl::MT, Tl::NT, kC, false, false>(acc, sT, LCb, sX, LKb, m0, n0);
    if (tcr) {  // token-row tile of the tensor-core pass
      const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
      for (int mt = 0; mt < Tl::MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < Tl::NT; ++nt)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int r = m0 + 16 * mt + g + 8 * hh, c = n0 + 8 * nt + 2 * t;
            *reinterpret_cast<__nv_bfloat162*>(prb + TcRec::oW + tile_off(r, c)) =
                __floats2bfloat162_rn(acc[mt][nt][2 * hh], acc[mt][nt][2 * hh + 1]);
          }
    } else {
      acc_to_bf16(acc, pr + PR::oW, PR::LKb, m0, n0);
    }
  }
  {  // U = T (beta v), fp32
    using Tl = Tiling<kC, DV>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4];
    zero(acc);
    warp_mma_bf16<Tl::MT, Tl::NT, kC, false, false>(acc, sT, LCb, sY, LMb, m0, n0);
    acc_to_global(acc, a.U + rec * kC * DV, DV, m0, n0);
  }
}

// ------------------------------------------------------------------ kernel 3 (bf16 operands)
// Two CTAs of 8 warps per SM: the tiles stay under half of the SM's shared
// memory by taking S0 and dS in halves of 64 key rows (the S0 half over the
// v tile once v is dead), so one CTA's barriers and loads overlap the other's
// products.
constexpr int kLaThreads = 256;
template <int DK, int DV>
struct LocalAPlanB {  // bytes
  static constexpr int LVb = DV + 8, LCb = kC + 8, HR = 64;  // HR: key rows per half of S0 / dS
  static constexpr size_t tv = (size_t)kC * LVb * 2;
  static constexpr size_t oO = 0, oVp = oO + tv, odV = oVp + tv, ov = odV + tv, oT = ov + tv,
                          odS = oT + (size_t)kC * LCb * 2, ob = odS + (size_t)HR * LVb * 2, ored = ob + kC * 4,
                          bytes = ored + 2 * kC * 4;
  static_assert((size_t)HR * LVb * 2 <= tv, "an S0 half fits over the v tile");
};

// Per chunk, bf16 inputs: the products that contract over the value channels,
// all operands bf16 images in shared memory (S0, dS, V', dV' and T come from
// the state passes and the prep kernel as bf16).
template <int DK, int DV>
__global__ void __launch_bounds__(kLaThreads, 2) bwd_local_a_bf16_kernel(const ChunkBwdArgs a) {
  pdl_wait();  // the previous kernel of the call has finished
  pdl_trigger();
  using PL = LocalAPlanB<DK, DV>;
  constexpr int LVb = PL::LVb, LCb = PL::LCb, HR = PL::HR, NTH = kLaThreads, NW = NTH / 32;
  extern __shared__ __align__(16) uint8_t smb[];
  bf16* sO = reinterpret_cast<bf16*>(smb + PL::oO);    // [64][LVb] dO
  bf16* sVp = reinterpret_cast<bf16*>(smb + PL::oVp);  // [64][LVb] V'
  bf16* sdV = reinterpret_cast<bf16*>(smb + PL::odV);  // [64][LVb] dV'
  bf16* sv = reinterpret_cast<bf16*>(smb + PL::ov);    // [64][LVb] v, then [HR][LVb] rows of S0
  bf16* sS0 = sv;
  bf16* sT = reinterpret_cast<bf16*>(smb + PL::oT);    // [64][LCb] T
  bf16* sdS = reinterpret_cast<bf16*>(smb + PL::odS);  // [HR][LVb] rows of dS
  float* sb = reinterpret_cast<float*>(smb + PL::ob);  // [64] beta
  float* red = reinterpret_cast<float*>(smb + PL::ored);  // [2][64] row sums per column group
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % a.NC, lb = blockIdx.x / a.NC, bh = a.bh0 + lb, t0 = n * kC, nv = min(kC, a.T - t0);
  const size_t row0 = row_of(a, bh, t0), rec = (size_t)lb * a.NC + n;
  // rows of 16-byte pieces: [rows][width] bf16 from global (row i at src_row(i)) into [rows][ld]
  auto rows_in = [&](bf16* dst, int ld, int rows, int width, auto src_row, int valid) {
    const int per = width / 8;
    for (int idx = tid; idx < rows * per; idx += NTH) {
      const int i = idx / per, c = (idx % per) * 8;
      cp16(dst + i * ld + c, i < valid ? src_row(i) + c : src_row(0), i < valid ? 16 : 0);
    }
  };
  const bf16* d_o = static_cast<const bf16*>(a.d_o);
  const bf16* vin = static_cast<const bf16*>(a.v);
  const bf16* Vp = reinterpret_cast<const bf16*>(a.Vp) + rec * kC * DV;
  const bf16* dVp = reinterpret_cast<const bf16*>(a.dVp) + rec * kC * DV;
  const bf16* S0 = reinterpret_cast<const bf16*>(a.S0c) + rec * DK * DV;
  const bf16* dS = reinterpret_cast<const bf16*>(a.dSc) + rec * DK * DV;
  const bf16* Tg = reinterpret_cast<const bf16*>(a.Tm) + rec * kC * kC;
  rows_in(sO, LVb, kC, DV, [&](int i) { return d_o + (row0 + (size_t)i * a.H) * DV; }, nv);
  rows_in(sv, LVb, kC, DV, [&](int i) { return vin + (row0 + (size_t)i * a.H) * DV; }, nv);
  rows_in(sVp, LVb, kC, DV, [&](int i) { return Vp + (size_t)i * DV; }, kC);
  rows_in(sdV, LVb, kC, DV, [&](int i) { return dVp + (size_t)i * DV; }, kC);
  rows_in(sT, LCb, kC, kC, [&](int i) { return Tg + (size_t)i * kC; }, kC);
  rows_in(sdS, LVb, HR, DV, [&](int i) { return dS + (size_t)i * DV; }, HR);  // first half of dS
  if (tid < kC) sb[tid] = tid < nv ? to_f32(static_cast<const bf16*>(a.beta)[row0 + (size_t)tid * a.H]) : 0.f;
  cp_wait();
  __syncthreads();
  {
    using Tl = Tiling<kC, kC, NW>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4];
    zero(acc);  // dAqk = tril(dO V'^T)
    warp_mma_bf16<Tl::MT, Tl::NT, DV, false, true>(acc, sO, LVb, sVp, LVb, m0, n0);
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int j) {
      if (j > i) acc[mt][nt][e] = 0.f;
    });
    acc_to_bf16(acc, reinterpret_cast<bf16*>(a.dAqk) + rec * kC * kC, kC, m0, n0);  // an operand only: bf16
    zero(acc);  // dU (beta V)^T, strictly lower part (bf16: the sum it enters is rounded to bf16 at once)
    warp_mma_bf16<Tl::MT, Tl::NT, DV, false, true>(acc, sdV, LVb, sv, LVb, m0, n0);
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int j) {
      acc[mt][nt][e] = j < i ? acc[mt][nt][e] * sb[j] : 0.f;
    });
    acc_to_bf16(acc, reinterpret_cast<bf16*>(a.dT1) + rec * kC * kC, kC, m0, n0);
  }
  {  // X = T^T dU: dv = beta X, dbeta part = rowsum(V . X)
    using Tl = Tiling<kC, DV, NW>;
    const int m0 = Tl::m0(warp), n0 = Tl::n0(warp);
    float acc[Tl::MT][Tl::NT][4], rp[Tl::MT][2] = {};
    zero(acc);
    warp_mma_bf16<Tl::MT, Tl::NT, kC, true, false>(acc, sT, LCb, sdV, LVb, m0, n0);
    bf16* dv = static_cast<bf16*>(a.dv);
    for_acc<Tl::MT, Tl::NT>(m0, n0, [&](int mt, int nt, int e, int i, int c) {
      const float x = acc[mt][nt][e];
      if (i < nv) dv[(row0 + (size_t)i * a.H) * DV + c] = __float2bfloat16_rn(sb[i] * x);
      rp[mt][e >> 1] = fmaf(x, __bfloat162float(sv[i * LVb + c]), rp[mt][e >> 1]);
    });
    row_sums_out<Tl::MT>(rp, m0, red + (warp / Tl::WM) * kC);
  }
  // dO S0^T, -dV' S0^T, V' dS^T (64 x DK, contracting the value channels) and
  // rowsum(dS . S0), by halves of HR key rows
  using Th = Tiling<kC, HR, NW>;
  const int hm0 = Th::m0(warp), hn0 = Th::n0(warp);
  for (int half = 0; half < DK / HR; ++half) {
    __syncthreads();  // v (or the previous halves) no longer read
    rows_in(sS0, LVb, HR, DV, [&](int i) { return S0 + (size_t)(half * HR + i) * DV; }, HR);
    if (half > 0) rows_in(sdS, LVb, HR, DV, [&](int i) { return dS + (size_t)(half * HR + i) * DV; }, HR);
    cp_wait();
    __syncthreads();
    float acc[Th::MT][Th::NT][4];
    zero(acc);
    warp_mma_bf16<Th::MT, Th::NT, DV, false, true>(acc, sO, LVb, sS0, LVb, hm0, hn0);
    acc_to_bf16(acc, reinterpret_cast<bf16*>(a.dQs) + rec * kC * DK + half * HR, DK, hm0, hn0);  // bf16 for the fold
    zero(acc);
    warp_mma_bf16<Th::MT, Th::NT, DV, false, true>(acc, sdV, LVb, sS0, LVb, hm0, hn0);
    for_acc<Th::MT, Th::NT>(hm0, hn0, [&](int mt, int nt, int e, int i, int c) { acc[mt][nt][e] = -acc[mt][nt][e]; });
    acc_to_bf16(acc, reinterpret_cast<bf16*>(a.dW) + rec * kC * DK + half * HR, DK, hm0, hn0);  // operand only
    zero(acc);
    warp_mma_bf16<Th::MT, Th::NT, DV, false, true>(acc, sVp, LVb, sdS, LVb, hm0, hn0);
    acc_to_bf16(acc, reinterpret_cast<bf16*>(a.dKb) + rec * kC * DK + half * HR, DK, hm0, hn0);  // bf16 for the fold
    for (int r = warp; r < HR; r += NW) {  // rowsum(dS . S0), two columns per load
      float x = 0.f;
      for (int c = 2 * lane; c < DV; c += 64) {
        const float2 d = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sdS + r * LVb + c));
        const float2 s0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(sS0 + r * LVb + c));
        x = fmaf(d.x, s0.x, fmaf(d.y, s0.y, x));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
      if (lane == 0) a.dgam[rec * DK + half * HR + r] = x;
    }
  }
  __syncthreads();
  if (tid < kC) {
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < Tiling<kC, DV, NW>::WN; ++w) x += red[w * kC + tid];
    a.dbu[rec * kC + tid] = x;
  }
}

// ------------------------------------------------------------------ kernel 4
template <int DK, int DV>
constexpr size_t local_b_smem() {
  constexpr int LK = DK + 4;
  return sizeof(float) * ((size_t)4 * kC * LK + 4 * kC * kLC + kC + 8 * kC + 4 * DK);
}

// Per chunk: dT, dA, the pairwise gradients and the fold into dq, dk, dg, dbeta.
template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1) bwd_local_b_kernel(const ChunkBwdArgs a) {
  pdl_wait();  // the previous kernel of the call has finished
  pdl_trigger();
  constexpr bool X3 = std::is_same<IO, float>::value;
  constexpr int LK = DK + 4;
  using TK = Tiling<kC, DK>;  // every 64 x d_k product: the same tile per warp
  using TC = Tiling<kC, kC>;
  extern __shared__ __align__(16) float sm[];
  float* sG = sm;               // [64][LK] cumulative log-gates
  float* sX = sG + kC * LK;     // [64][LK] K+, then K+_r (exact path: k), then dG
  float* sY = sX + kC * LK;     // [64][LK] dW, then K-_r
  float* sZ = sY + kC * LK;     // [64][LK] Q+_r (exact path: scale q)
  float* sT = sZ + kC * LK;     // [64][kLC] T
  float* sDT = sT + kC * kLC;   // [64][kLC] dT, then M = diag(beta) dA
  float* sY2 = sDT + kC * kLC;  // [64][kLC] dT T^T
  float* sQA = sY2 + kC * kLC;  // [64][kLC] dAqk
  float* sb = sQA + kC * kLC;   // [64] beta
  float* red = sb + kC;         // [8][64] row sums per column group: K+ . T^T dW (slots 0-3), dA . P (4-7)
  float* colC = red + 8 * kC;   // [4][DK] column sums of dKbar . Kbar per row group
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % a.NC, lb = blockIdx.x / a.NC, bh = a.bh0 + lb, t0 = n * kC, nv = min(kC, a.T - t0);
  const size_t row0 = row_of(a, bh, t0), rec = (size_t)lb * a.NC + n;
  const IO* q = static_cast<const IO*>(a.q);
  const IO* k = static_cast<const IO*>(a.k);
  const int m0 = TK::m0(warp), n0 = TK::n0(warp), cm0 = TC::m0(warp), cn0 = TC::n0(warp);
  float dk_acc[TK::MT][TK::NT][4], dG_acc[TK::MT][TK::NT][4];
  zero(dk_acc);
  zero(dG_acc);

  if (tid < kC) sb[tid] = tid < nv ? to_f32(static_cast<const IO*>(a.beta)[row0 + (size_t)tid * a.H]) : 0.f;
  const bool slow = load_gates_cumsum<IO, DK>(sG, LK, static_cast<const IO*>(a.g), a.gate, row0, a.H, nv);
  load_rows<IO, DK>(sX, LK, k, row0, a.H, nv, DK, 0);
  load_f32(sY, LK, a.dW + rec * kC * DK, DK, kC, DK);
  load_f32(sT, kLC, a.Tm + rec * kC * kC, kC, kC, kC);
  load_f32(sDT, kLC, a.dT1 + rec * kC * kC, kC, kC, kC);
  cp_wait();
  __syncthreads();
  for (int idx = tid; idx < kC * DK; idx += kThreads) {
    const int i = idx / DK, r = idx % DK;
    sX[i * LK + r] *= expf(sG[i * LK + r]);
  }
  __syncthreads();
  {  // dT += dW (beta K+)^T, strictly lower part
    float acc[TC::MT][TC::NT][4];
    zero(acc);
    warp_mma_kk<TC::MT, TC::NT, X3, DK>(acc, sY, LK, sX, LK, cm0, cn0);
    for_acc<TC::MT, TC::NT>(cm0, cn0, [&](int mt, int nt, int e, int i, int j) {
      if (j < i) sDT[i * kLC + j] += acc[mt][nt][e] * sb[j];
    });
  }
  {  // X = T^T dW: dK+ = beta X; dbeta part rowsum(K+ . X)
    float acc[TK::MT][TK::NT][4], rp[TK::MT][2] = {};
    zero(acc);
    warp_mma<TK::MT, TK::NT, X3, kC>(acc, colm(sT, kLC), rowm(sY, LK), m0, n0);
    for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
      const float x = acc[mt][nt][e], kp = sX[i * LK + r], bx = sb[i] * x;
      dk_acc[mt][nt][e] = fmaf(bx, expf(sG[i * LK + r]), dk_acc[mt][nt][e]);
      dG_acc[mt][nt][e] = fmaf(bx, kp, dG_acc[mt][nt][e]);
      rp[mt][e >> 1] = fmaf(x, kp, rp[mt][e >> 1]);
    });
    row_sums_out<TK::MT>(rp, m0, red + (warp / TK::WM) * kC);
  }
  __syncthreads();
  {  // dT T^T
    float acc[TC::MT][TC::NT][4];
    zero(acc);
    warp_mma_kk<TC::MT, TC::NT, X3, kC>(acc, sDT, kLC, sT, kLC, cm0, cn0);
    for_acc<TC::MT, TC::NT>(cm0, cn0,
                            [&](int mt, int nt, int e, int i, int j) { sY2[i * kLC + j] = acc[mt][nt][e]; });
  }
  __syncthreads();
  {  // dA = -T^T (dT T^T), strictly lower; dbeta part rowsum(dA . P); M = diag(beta) dA
    float acc[TC::MT][TC::NT][4], rp[TC::MT][2] = {};
    zero(acc);
    warp_mma<TC::MT, TC::NT, X3, kC>(acc, colm(sT, kLC), rowm(sY2, kLC), cm0, cn0);
    const float* P = a.Pkk + rec * kC * kC;
    for_acc<TC::MT, TC::NT>(cm0, cn0, [&](int mt, int nt, int e, int i, int j) {
      const float d = j < i ? -acc[mt][nt][e] : 0.f;
      rp[mt][e >> 1] = fmaf(d, P[i * kC + j], rp[mt][e >> 1]);
      sDT[i * kLC + j] = sb[i] * d;
    });
    row_sums_out<TC::MT>(rp, cm0, red + (4 + warp / TC::WM) * kC);
  }
  // operands of the pairwise gradients
  load_f32(sQA, kLC, a.dAqk + rec * kC * kC, kC, kC, kC);
  load_rows<IO, DK>(sX, LK, k, row0, a.H, nv, DK, 0);
  load_rows<IO, DK>(sZ, LK, q, row0, a.H, nv, DK, 0);
  cp_wait();
  __syncthreads();
  for (int idx = tid; idx < kC * DK; idx += kThreads) {
    const int i = idx / DK, r = idx % DK;
    const float kk = sX[i * LK + r], qq = a.scale * sZ[i * LK + r];
    if (!slow) {
      const float d = sG[i * LK + r] - sG[kRef * LK + r], ex = expf(d);
      sX[i * LK + r] = kk * ex;
      sY[i * LK + r] = kk * expf(-d);
      sZ[i * LK + r] = qq * ex;
    } else {
      sZ[i * LK + r] = qq;
    }
  }
  __syncthreads();
  const float* dQs = a.dQs + rec * kC * DK;
  const float* Qp = a.Qp + rec * kC * DK;
  IO* dq = static_cast<IO*>(a.dq);
  if (!slow) {
    {  // dQ+_r = dAqk K-_r;  dq = scale (exp(G - G_ref) dQ+_r + Gamma dO S0^T)
      float acc[TK::MT][TK::NT][4];
      zero(acc);
      warp_mma<TK::MT, TK::NT, X3, kC>(acc, rowm(sQA, kLC), rowm(sY, LK), m0, n0);
      for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
        const float x = acc[mt][nt][e], G = sG[i * LK + r];
        const float ex = expf(G - sG[kRef * LK + r]), dqs = dQs[i * DK + r];
        if (i < nv) dq[(row0 + (size_t)i * a.H) * DK + r] = from_f32<IO>(a.scale * fmaf(ex, x, expf(G) * dqs));
        dG_acc[mt][nt][e] += fmaf(x, sZ[i * LK + r], dqs * Qp[i * DK + r]);
      });
    }
    {  // dK-_r = dAqk^T Q+_r + M^T K+_r
      float acc[TK::MT][TK::NT][4];
      zero(acc);
      warp_mma<TK::MT, TK::NT, X3, kC>(acc, colm(sQA, kLC), rowm(sZ, LK), m0, n0);
      warp_mma<TK::MT, TK::NT, X3, kC>(acc, colm(sDT, kLC), rowm(sX, LK), m0, n0);
      for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
        const float x = acc[mt][nt][e];
        dk_acc[mt][nt][e] = fmaf(expf(sG[kRef * LK + r] - sG[i * LK + r]), x, dk_acc[mt][nt][e]);
        dG_acc[mt][nt][e] = fmaf(-x, sY[i * LK + r], dG_acc[mt][nt][e]);
      });
    }
    {  // dK+_r = M K-_r
      float acc[TK::MT][TK::NT][4];
      zero(acc);
      warp_mma<TK::MT, TK::NT, X3, kC>(acc, rowm(sDT, kLC), rowm(sY, LK), m0, n0);
      for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
        const float x = acc[mt][nt][e];
        dk_acc[mt][nt][e] = fmaf(expf(sG[i * LK + r] - sG[kRef * LK + r]), x, dk_acc[mt][nt][e]);
        dG_acc[mt][nt][e] = fmaf(x, sX[i * LK + r], dG_acc[mt][nt][e]);
      });
    }
  } else {
    // exact pairwise terms, E = exp(G_ir - G_jr) for j <= i:
    //   Aqk_ij = sum_r (scale q_ir) k_jr E,  P_ij = sum_r k_ir k_jr E
    for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
      const float Gi = sG[i * LK + r], ki = sX[i * LK + r], qi = sZ[i * LK + r];
      float dqp = 0.f, dkp = 0.f, dgp = 0.f;
      for (int j = 0; j <= i; ++j) {  // row i of dAqk and M: i is the left factor
        const float kE = expf(Gi - sG[j * LK + r]) * sX[j * LK + r];
        const float c = sQA[i * kLC + j], m = sDT[i * kLC + j];
        dqp = fmaf(c, kE, dqp);
        dkp = fmaf(m, kE, dkp);
        dgp = fmaf(fmaf(c, qi, m * ki), kE, dgp);
      }
      for (int j = i; j < kC; ++j) {  // column i of dAqk and M: i is the right factor
        const float w =
            fmaf(sQA[j * kLC + i], sZ[j * LK + r], sDT[j * kLC + i] * sX[j * LK + r]) * expf(sG[j * LK + r] - Gi);
        dkp += w;
        dgp = fmaf(-w, ki, dgp);
      }
      const float dqs = dQs[i * DK + r];
      if (i < nv) dq[(row0 + (size_t)i * a.H) * DK + r] = from_f32<IO>(a.scale * fmaf(expf(Gi), dqs, dqp));
      dk_acc[mt][nt][e] += dkp;
      dG_acc[mt][nt][e] += fmaf(dqs, Qp[i * DK + r], dgp);
    });
  }
  {  // Kbar: dk += exp(G_C - G) dKbar, dG -= dKbar . Kbar, dG_C += column sums of the same
    const float* dKb = a.dKb + rec * kC * DK;
    const float* Kb = a.Kb + rec * kC * DK;
    float cp[TK::MT][TK::NT][2] = {};
    for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
      const float x = dKb[i * DK + r], y = x * Kb[i * DK + r];
      dk_acc[mt][nt][e] = fmaf(expf(sG[(kC - 1) * LK + r] - sG[i * LK + r]), x, dk_acc[mt][nt][e]);
      dG_acc[mt][nt][e] -= y;
      cp[mt][nt][e & 1] += y;
    });
#pragma unroll
    for (int nt = 0; nt < TK::NT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float x = 0.f;
#pragma unroll
        for (int mt = 0; mt < TK::MT; ++mt) x += cp[mt][nt][c];
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        if (lane < 4) colC[(warp % TK::WM) * DK + n0 + 8 * nt + 2 * lane + c] = x;
      }
  }
  IO* dk = static_cast<IO*>(a.dk);
  for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
    if (i < nv) dk[(row0 + (size_t)i * a.H) * DK + r] = from_f32<IO>(dk_acc[mt][nt][e]);
  });
  __syncthreads();  // sX is no longer read: it takes dG
  for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) { sX[i * LK + r] = dG_acc[mt][nt][e]; });
  __syncthreads();
  if (tid < DK) {  // the dG_C terms of channel r, into colC row 0
    const int r = tid;
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < TK::WM; ++w) x += colC[w * DK + r];
    colC[r] = fmaf(expf(sG[(kC - 1) * LK + r]), a.dgam[rec * DK + r], x);
  }
  __syncthreads();
  if (tid < DK) {  // dg = reverse cumsum of dG over the chunk, plus the dG_C terms
    float acc = colC[tid];
    for (int i = kC - 1; i >= 0; --i) {
      acc += sX[i * LK + tid];
      sX[i * LK + tid] = acc;
    }
  }
  __syncthreads();
  if (a.gate == KDA_GATE_CHANNEL) {
    IO* dg = static_cast<IO*>(a.dg);
    for (int idx = tid; idx < nv * DK; idx += kThreads) {
      const int i = idx / DK, r = idx % DK;
      dg[(row0 + (size_t)i * a.H) * DK + r] = from_f32<IO>(sX[i * LK + r]);
    }
  } else if (a.gate == KDA_GATE_HEAD) {
    IO* dg = static_cast<IO*>(a.dg);
    for (int i = warp; i < nv; i += kThreads / 32) {
      float x = 0.f;
      for (int r = lane; r < DK; r += 32) x += sX[i * LK + r];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
      if (lane == 0) dg[row0 + (size_t)i * a.H] = from_f32<IO>(x);
    }
  }
  if (tid < nv) {
    float x = a.dbu[rec * kC + tid], y = 0.f;
#pragma unroll
    for (int w = 0; w < TK::WN; ++w) x += red[w * kC + tid];
#pragma unroll
    for (int w = 0; w < TC::WN; ++w) y += red[(4 + w) * kC + tid];
    static_cast<IO*>(a.dbeta)[row0 + (size_t)tid * a.H] = from_f32<IO>(x + y);
  }
}


// ------------------------------------------------------------------ kernel 4 (bf16 operands)
template <int DK, int DV>
struct LocalBPlanB {  // bytes
  static constexpr int LK = DK + 4, LKb = DK + 8, LCb = kC + 8;
  static constexpr size_t tk = (size_t)kC * LKb * 2, tc = (size_t)kC * LCb * 2;
  static constexpr size_t oG = 0, ok = oG + (size_t)kC * LK * 4, oq = ok + tk, oA = oq + tk, oB = oA + tk,
                          oC = oB + tk, oT = oC + tk, oDT = oT + tc, oY = oDT + tc, oQA = oY + tc, ob = oQA + tc,
                          ored = ob + kC * 4, ocol = ored + 8 * kC * 4, oQs = ocol + 4 * DK * 4,
                          oKs = oQs + tk, oD1 = oKs + tk, oPk = oD1 + tc, bytes = oPk + (size_t)kC * kLC * 4;
  static_assert(tk % 16 == 0 && tc % 16 == 0 && ok % 16 == 0, "16 B");
  static_assert(2 * tk >= (size_t)kC * LK * 4, "dG (fp32) fits over the k and q tiles");
};

// Per chunk, bf16 inputs: dT, T^T dW, dA, the pairwise gradients and the fold
// into dq, dk, dg, dbeta.  Operands are bf16 images; G, the decay factors and
// the fold run in fp32 (from the exact k, q inputs), exponentials by the fast
// intrinsic (exponents bounded by the factored form's span, or <= 0).
template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1) bwd_local_b_bf16_kernel(const ChunkBwdArgs a) {
  pdl_wait();  // the previous kernel of the call has finished
  pdl_trigger();
  using PL = LocalBPlanB<DK, DV>;
  constexpr int LK = PL::LK, LKb = PL::LKb, LCb = PL::LCb;
  using TK = Tiling<kC, DK>;  // every 64 x d_k product: the same tile per warp
  using TC = Tiling<kC, kC>;
  extern __shared__ __align__(16) uint8_t smb[];
  float* sG = reinterpret_cast<float*>(smb + PL::oG);   // [64][LK] cumulative log-gates
  bf16* sk = reinterpret_cast<bf16*>(smb + PL::ok);     // [64][LKb] k (input)
  bf16* sq = reinterpret_cast<bf16*>(smb + PL::oq);     // [64][LKb] q (input)
  bf16* sA = reinterpret_cast<bf16*>(smb + PL::oA);     // [64][LKb] dW, then K-_r
  bf16* sB = reinterpret_cast<bf16*>(smb + PL::oB);     // [64][LKb] K+, then K+_r
  bf16* sC = reinterpret_cast<bf16*>(smb + PL::oC);     // [64][LKb] Q+_r
  bf16* sT = reinterpret_cast<bf16*>(smb + PL::oT);     // [64][LCb] T
  bf16* sDT = reinterpret_cast<bf16*>(smb + PL::oDT);   // [64][LCb] dT, then M = diag(beta) dA
  bf16* sY = reinterpret_cast<bf16*>(smb + PL::oY);     // [64][LCb] dT T^T
  bf16* sQA = reinterpret_cast<bf16*>(smb + PL::oQA);   // [64][LCb] dAqk
  float* sb = reinterpret_cast<float*>(smb + PL::ob);   // [64] beta
  float* red = reinterpret_cast<float*>(smb + PL::ored);  // [8][64] row sums per column group
  float* colC = reinterpret_cast<float*>(smb + PL::ocol);  // [4][DK] column sums of dKbar . Kbar
  float* sdG = reinterpret_cast<float*>(smb + PL::ok);  // [64][LK] dG (fp32), over the k and q tiles at the end
  bf16* sQs = reinterpret_cast<bf16*>(smb + PL::oQs);  // [64][LKb] dO S0^T (bf16, from the d_v kernel)
  bf16* sKs = reinterpret_cast<bf16*>(smb + PL::oKs);  // [64][LKb] dKbar (bf16, from the d_v kernel)
  bf16* sD1 = reinterpret_cast<bf16*>(smb + PL::oD1);  // [64][LCb] dU (beta V)^T (bf16, from the d_v kernel)
  float* sPk = reinterpret_cast<float*>(smb + PL::oPk);  // [64][kLC] P (fp32, from the preparation)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = blockIdx.x % a.NC, lb = blockIdx.x / a.NC, bh = a.bh0 + lb, t0 = n * kC, nv = min(kC, a.T - t0);
  const size_t row0 = row_of(a, bh, t0), rec = (size_t)lb * a.NC + n;
  const bf16* q = static_cast<const bf16*>(a.q);
  const bf16* k = static_cast<const bf16*>(a.k);
  const int m0 = TK::m0(warp), n0 = TK::n0(warp), cm0 = TC::m0(warp), cn0 = TC::n0(warp);
  float dk_acc[TK::MT][TK::NT][4], dG_acc[TK::MT][TK::NT][4];
  zero(dk_acc);
  zero(dG_acc);
  auto rows_in = [&](bf16* dst, const bf16* src) {  // 64 input rows of DK (zeros past the tail)
    constexpr int per = DK / 8;
    for (int idx = tid; idx < kC * per; idx += kThreads) {
      const int i = idx / per, c = (idx % per) * 8;
      cp16(dst + i * LKb + c, i < nv ? src + (row0 + (size_t)i * a.H) * DK + c : src, i < nv ? 16 : 0);
    }
  };


  if (tid < kC) sb[tid] = tid < nv ? to_f32(static_cast<const bf16*>(a.beta)[row0 + (size_t)tid * a.H]) : 0.f;
  rows_in(sk, k);
  rows_in(sq, q);
  const bool slow = load_gates_cumsum<bf16, DK>(sG, LK, static_cast<const bf16*>(a.g), a.gate, row0, a.H, nv);
  {  // dW and dAqk (bf16 from the d_v kernel)
    const bf16* dWg = reinterpret_cast<const bf16*>(a.dW) + rec * kC * DK;
    const bf16* dAg = reinterpret_cast<const bf16*>(a.dAqk) + rec * kC * kC;
    for (int idx = tid; idx < kC * (DK / 8); idx += kThreads) {
      const int i = idx / (DK / 8), c = (idx % (DK / 8)) * 8;
      cp16(sA + i * LKb + c, dWg + (size_t)i * DK + c, 16);
    }
    for (int idx = tid; idx < kC * (kC / 8); idx += kThreads) {
      const int i = idx / (kC / 8), c = (idx % (kC / 8)) * 8;
      cp16(sQA + i * LCb + c, dAg + (size_t)i * kC + c, 16);
    }
  }
  {
    const bf16* Tg = reinterpret_cast<const bf16*>(a.Tm) + rec * kC * kC;
    const bf16* D1g = reinterpret_cast<const bf16*>(a.dT1) + rec * kC * kC;
    for (int idx = tid; idx < kC * (kC / 8); idx += kThreads) {
      const int i = idx / (kC / 8), c = (idx % (kC / 8)) * 8;
      cp16(sT + i * LCb + c, Tg + (size_t)i * kC + c, 16);
      cp16(sD1 + i * LCb + c, D1g + (size_t)i * kC + c, 16);
    }
    const float* Pg = a.Pkk + rec * kC * kC;
    for (int idx = tid; idx < kC * (kC / 4); idx += kThreads) {
      const int i = idx / (kC / 4), c = (idx % (kC / 4)) * 4;
      cp16(sPk + i * kLC + c, Pg + (size_t)i * kC + c, 16);
    }
  }
  cp_commit();  // group 1: everything the products and their epilogues need
  {  // group 2: the fold's inputs, in flight while the products run (rows padded against bank conflicts)
    const bf16* qs = reinterpret_cast<const bf16*>(a.dQs) + rec * kC * DK;
    const bf16* ks = reinterpret_cast<const bf16*>(a.dKb) + rec * kC * DK;
    for (int idx = tid; idx < kC * (DK / 8); idx += kThreads) {
      const int i = idx / (DK / 8), c = (idx % (DK / 8)) * 8;
      cp16(sQs + i * LKb + c, qs + (size_t)i * DK + c, 16);
      cp16(sKs + i * LKb + c, ks + (size_t)i * DK + c, 16);
    }
  }
  cp_commit();
  cp_wait_group<1>();
  __syncthreads();
  // 8 channels of a row per step: 16-byte bf16 and fp32 shared-memory accesses
  auto ld8f = [](const float* p, float* f) {
    const float4 a0 = *reinterpret_cast<const float4*>(p), a1 = *reinterpret_cast<const float4*>(p + 4);
    f[0] = a0.x, f[1] = a0.y, f[2] = a0.z, f[3] = a0.w, f[4] = a1.x, f[5] = a1.y, f[6] = a1.z, f[7] = a1.w;
  };
  auto ld8b = [](const bf16* p, float* f) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
      f[2 * e] = t.x, f[2 * e + 1] = t.y;
    }
  };
  auto st8b = [](bf16* p, const float* f) {
    uint32_t u[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 t = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
      u[e] = *reinterpret_cast<const uint32_t*>(&t);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(u[0], u[1], u[2], u[3]);
  };
  for (int idx = tid; idx < kC * (DK / 8); idx += kThreads) {  // K+ = k exp(G)
    const int i = idx / (DK / 8), r = (idx % (DK / 8)) * 8;
    float kk[8], G[8], w[8];
    ld8b(sk + i * LKb + r, kk);
    ld8f(sG + i * LK + r, G);
#pragma unroll
    for (int e = 0; e < 8; ++e) w[e] = kk[e] * __expf(G[e]);
    st8b(sB + i * LKb + r, w);
  }
  __syncthreads();
  {  // dT = dU (beta V)^T + dW (beta K+)^T, strictly lower, as a bf16 image
    float acc[TC::MT][TC::NT][4];
    zero(acc);
    warp_mma_bf16<TC::MT, TC::NT, DK, false, true>(acc, sA, LKb, sB, LKb, cm0, cn0);
    for_acc<TC::MT, TC::NT>(cm0, cn0, [&](int mt, int nt, int e, int i, int j) {
      acc[mt][nt][e] = j < i ? fmaf(acc[mt][nt][e], sb[j], __bfloat162float(sD1[i * LCb + j])) : 0.f;
    });
    acc_to_bf16(acc, sDT, LCb, cm0, cn0);
  }
  {  // X = T^T dW: dK+ = beta X; dbeta part rowsum(K+ . X)
    float acc[TK::MT][TK::NT][4], rp[TK::MT][2] = {};
    zero(acc);
    warp_mma_bf16<TK::MT, TK::NT, kC, true, false>(acc, sT, LCb, sA, LKb, m0, n0);
    for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
      const float x = acc[mt][nt][e], gm = __expf(sG[i * LK + r]);
      const float kp = __bfloat162float(sk[i * LKb + r]) * gm, bx = sb[i] * x;
      dk_acc[mt][nt][e] = fmaf(bx, gm, dk_acc[mt][nt][e]);
      dG_acc[mt][nt][e] = fmaf(bx, kp, dG_acc[mt][nt][e]);
      rp[mt][e >> 1] = fmaf(x, kp, rp[mt][e >> 1]);
    });
    row_sums_out<TK::MT>(rp, m0, red + (warp / TK::WM) * kC);
  }
  __syncthreads();
  {  // dT T^T
    float acc[TC::MT][TC::NT][4];
    zero(acc);
    warp_mma_bf16<TC::MT, TC::NT, kC, false, true>(acc, sDT, LCb, sT, LCb, cm0, cn0);
    acc_to_bf16(acc, sY, LCb, cm0, cn0);
  }
  __syncthreads();
  {  // dA = -T^T (dT T^T), strictly lower; dbeta part rowsum(dA . P); M = diag(beta) dA
    float acc[TC::MT][TC::NT][4], rp[TC::MT][2] = {};
    zero(acc);
    warp_mma_bf16<TC::MT, TC::NT, kC, true, false>(acc, sT, LCb, sY, LCb, cm0, cn0);
    for_acc<TC::MT, TC::NT>(cm0, cn0, [&](int mt, int nt, int e, int i, int j) {
      const float d = j < i ? -acc[mt][nt][e] : 0.f;
      rp[mt][e >> 1] = fmaf(d, sPk[i * kLC + j], rp[mt][e >> 1]);
      acc[mt][nt][e] = sb[i] * d;
    });
    acc_to_bf16(acc, sDT, LCb, cm0, cn0);
    row_sums_out<TC::MT>(rp, cm0, red + (4 + warp / TC::WM) * kC);
  }
  if (!slow) {  // factored operands K+_r, K-_r, Q+_r
    for (int idx = tid; idx < kC * (DK / 8); idx += kThreads) {
      const int i = idx / (DK / 8), r = (idx % (DK / 8)) * 8;
      float G[8], Gr[8], kk[8], qq[8], w[8], ex[8];
      ld8f(sG + i * LK + r, G);
      ld8f(sG + kRef * LK + r, Gr);
      ld8b(sk + i * LKb + r, kk);
      ld8b(sq + i * LKb + r, qq);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        G[e] -= Gr[e];  // d = G - G_ref
        ex[e] = __expf(G[e]);
        w[e] = kk[e] * ex[e];
      }
      st8b(sB + i * LKb + r, w);
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = kk[e] * __expf(-G[e]);
      st8b(sA + i * LKb + r, w);
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = (a.scale * qq[e]) * ex[e];
      st8b(sC + i * LKb + r, w);
    }
  }
  cp_wait_group<0>();  // the fold's inputs
  __syncthreads();
  auto dqs_at = [&](int i, int r) { return __bfloat162float(sQs[i * LKb + r]); };
  auto dkb_at = [&](int i, int r) { return __bfloat162float(sKs[i * LKb + r]); };
  float cp[TK::MT][TK::NT][2] = {};  // column partial sums of dKbar . Kbar (for dG_C)
  bf16* dq = static_cast<bf16*>(a.dq);
  if (!slow) {
    // the three pairwise products first, then one pass over the elements with
    // the decay factors taken once: ex = exp(G - G_ref), 1/ex, Gamma = exp(G)
    float aq[TK::MT][TK::NT][4], am[TK::MT][TK::NT][4], ap[TK::MT][TK::NT][4];
    zero(aq);  // dQ+_r = dAqk K-_r
    warp_mma_bf16<TK::MT, TK::NT, kC, false, false>(aq, sQA, LCb, sA, LKb, m0, n0);
    zero(am);  // dK-_r = dAqk^T Q+_r + M^T K+_r
    warp_mma_bf16<TK::MT, TK::NT, kC, true, false>(am, sQA, LCb, sC, LKb, m0, n0);
    warp_mma_bf16<TK::MT, TK::NT, kC, true, false>(am, sDT, LCb, sB, LKb, m0, n0);
    zero(ap);  // dK+_r = M K-_r
    warp_mma_bf16<TK::MT, TK::NT, kC, false, false>(ap, sDT, LCb, sA, LKb, m0, n0);
    for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
      const float G = sG[i * LK + r], d = G - sG[kRef * LK + r];
      const float ex = __expf(d), ei = __expf(-d), gm = __expf(G), dqs = dqs_at(i, r);
      const float kbf = __expf(sG[(kC - 1) * LK + r] - G);  // Kbar = k kbf
      const float kk = __bfloat162float(sk[i * LKb + r]);
      const float qs = a.scale * __bfloat162float(sq[i * LKb + r]);  // Q+_r = qs ex, Q+ = qs Gamma
      const float xq = aq[mt][nt][e], xm = am[mt][nt][e], xp = ap[mt][nt][e];
      if (i < nv) {  // dq = scale (exp(G - G_ref) dQ+_r + Gamma dO S0^T)
        const float v = a.scale * fmaf(ex, xq, gm * dqs);
        const size_t o = (row0 + (size_t)i * a.H) * DK + r;
        if (a.dq32) a.dq32[o] = v; else dq[o] = __float2bfloat16_rn(v);
      }
      const float xb = dkb_at(i, r), yb = xb * kk * kbf;  // the Kbar terms
      dk_acc[mt][nt][e] = fmaf(kbf, xb, fmaf(ei, xm, fmaf(ex, xp, dk_acc[mt][nt][e])));
      dG_acc[mt][nt][e] += fmaf(qs, fmaf(xq, ex, dqs * gm), kk * fmaf(xp, ex, -xm * ei)) - yb;
      cp[mt][nt][e & 1] += yb;
    });
  } else {
    // exact pairwise terms, E = exp(G_ir - G_jr) for j <= i (see the fp32 kernel)
    auto K_ = [&](int i, int r) { return __bfloat162float(sk[i * LKb + r]); };
    auto Q_ = [&](int i, int r) { return a.scale * __bfloat162float(sq[i * LKb + r]); };
    auto QA = [&](int i, int j) { return __bfloat162float(sQA[i * LCb + j]); };
    auto MM = [&](int i, int j) { return __bfloat162float(sDT[i * LCb + j]); };
    for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
      const float Gi = sG[i * LK + r], ki = K_(i, r), qi = Q_(i, r);
      float dqp = 0.f, dkp = 0.f, dgp = 0.f;
      for (int j = 0; j <= i; ++j) {
        const float kE = __expf(Gi - sG[j * LK + r]) * K_(j, r);
        const float c = QA(i, j), m = MM(i, j);
        dqp = fmaf(c, kE, dqp);
        dkp = fmaf(m, kE, dkp);
        dgp = fmaf(fmaf(c, qi, m * ki), kE, dgp);
      }
      for (int j = i; j < kC; ++j) {
        const float w = fmaf(QA(j, i), Q_(j, r), MM(j, i) * K_(j, r)) * __expf(sG[j * LK + r] - Gi);
        dkp += w;
        dgp = fmaf(-w, ki, dgp);
      }
      const float dqs = dqs_at(i, r), gm = __expf(Gi);
      if (i < nv) {
        const float v = a.scale * fmaf(gm, dqs, dqp);
        const size_t o = (row0 + (size_t)i * a.H) * DK + r;
        if (a.dq32) a.dq32[o] = v; else dq[o] = __float2bfloat16_rn(v);
      }
      dk_acc[mt][nt][e] += dkp;
      dG_acc[mt][nt][e] += fmaf(dqs, qi * gm, dgp);
    });
  }
  {  // Kbar: dk += exp(G_C - G) dKbar, dG -= dKbar . Kbar, dG_C += column sums of the same
    if (slow)  // (the fast path folded these into its epilogue)
      for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
        const float kbf = __expf(sG[(kC - 1) * LK + r] - sG[i * LK + r]);  // Kbar = k kbf
        const float x = dkb_at(i, r), y = x * __bfloat162float(sk[i * LKb + r]) * kbf;
        dk_acc[mt][nt][e] = fmaf(kbf, x, dk_acc[mt][nt][e]);
        dG_acc[mt][nt][e] -= y;
        cp[mt][nt][e & 1] += y;
      });
#pragma unroll
    for (int nt = 0; nt < TK::NT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float x = 0.f;
#pragma unroll
        for (int mt = 0; mt < TK::MT; ++mt) x += cp[mt][nt][c];
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        if (lane < 4) colC[(warp % TK::WM) * DK + n0 + 8 * nt + 2 * lane + c] = x;
      }
  }
  bf16* dk = static_cast<bf16*>(a.dk);
  for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) {
    if (i < nv) {
      const size_t o = (row0 + (size_t)i * a.H) * DK + r;
      if (a.dk32) a.dk32[o] = dk_acc[mt][nt][e]; else dk[o] = __float2bfloat16_rn(dk_acc[mt][nt][e]);
    }
  });
  __syncthreads();  // the k and q tiles are no longer read: they take dG
  for_acc<TK::MT, TK::NT>(m0, n0, [&](int mt, int nt, int e, int i, int r) { sdG[i * LK + r] = dG_acc[mt][nt][e]; });
  __syncthreads();
  if (tid < DK) {  // the dG_C terms of channel r, into colC row 0
    const int r = tid;
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < TK::WM; ++w) x += colC[w * DK + r];
    colC[r] = fmaf(__expf(sG[(kC - 1) * LK + r]), a.dgam[rec * DK + r], x);
  }
  __syncthreads();
  if (tid < DK) {  // dg = reverse cumsum of dG over the chunk, plus the dG_C terms
    float acc = colC[tid];
    for (int i = kC - 1; i >= 0; --i) {
      acc += sdG[i * LK + tid];
      sdG[i * LK + tid] = acc;
    }
  }
  __syncthreads();
  if (a.gate == KDA_GATE_CHANNEL) {
    bf16* dg = static_cast<bf16*>(a.dg);
    for (int idx = tid; idx < nv * DK; idx += kThreads) {
      const int i = idx / DK, r = idx % DK;
      dg[(row0 + (size_t)i * a.H) * DK + r] = __float2bfloat16_rn(sdG[i * LK + r]);
    }
  } else if (a.gate == KDA_GATE_HEAD) {
    bf16* dg = static_cast<bf16*>(a.dg);
    for (int i = warp; i < nv; i += kWarps) {
      float x = 0.f;
      for (int r = lane; r < DK; r += 32) x += sdG[i * LK + r];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
      if (lane == 0) dg[row0 + (size_t)i * a.H] = __float2bfloat16_rn(x);
    }
  }
  if (tid < nv) {
    float x = a.dbu[rec * kC + tid], y = 0.f;
#pragma unroll
    for (int w = 0; w < TK::WN; ++w) x += red[w * kC + tid];
#pragma unroll
    for (int w = 0; w < TC::WN; ++w) y += red[(4 + w) * kC + tid];
    static_cast<bf16*>(a.dbeta)[row0 + (size_t)tid * a.H] = __float2bfloat16_rn(x + y);
  }
}

// ------------------------------------------------------------------ host
// Floats of each workspace array per chunk record, in layout order.
struct WsPlan {
  size_t W, U, Qp, Kb, Wt, Qpt, Kbt, Aqk, prec, Tm, Pkk, gam, S0c, dSc, Vp, dVp, dAqk, dT1, dQs, dW, dKb, dgam, dbu;
  // fp32 inputs keep the passes' operands as fp32 arrays, bf16 inputs as one bf16 record per chunk
  explicit WsPlan(int dk, int dv, bool f32)
      : W(f32 ? (size_t)kC * dk : 0), U((size_t)kC * dv), Qp(f32 ? (size_t)kC * dk : 0), Kb(f32 ? (size_t)kC * dk : 0),
        Wt(f32 ? (size_t)kC * dk : 0), Qpt(f32 ? (size_t)kC * dk : 0), Kbt(f32 ? (size_t)kC * dk : 0),
        Aqk(f32 ? kC * kC : 0), prec(f32 ? 0 : (dk == 128 ? PassRec<128>::n : PassRec<64>::n) / 2),
        // bf16 inputs: T, S0, dS, V', dV', dAqk, dU (beta V)^T, dW, dO S0^T and dKbar are kept as bf16 (half the floats)
        Tm(kC * kC / (f32 ? 1 : 2)), Pkk(kC * kC), gam(dk), S0c((size_t)dk * dv / (f32 ? 1 : 2)), dSc((size_t)dk * dv / (f32 ? 1 : 2)),
        Vp((size_t)kC * dv / (f32 ? 1 : 2)), dVp((size_t)kC * dv / (f32 ? 1 : 2)), dAqk(kC * kC / (f32 ? 1 : 2)), dT1(kC * kC / (f32 ? 1 : 2)), dQs((size_t)kC * dk / (f32 ? 1 : 2)), dW((size_t)kC * dk / (f32 ? 1 : 2)),
        dKb((size_t)kC * dk / (f32 ? 1 : 2)), dgam(dk), dbu(kC) {}
  size_t per_rec() const {
    return W + U + Qp + Kb + Wt + Qpt + Kbt + Aqk + prec + Tm + Pkk + gam + S0c + dSc + Vp + dVp + dAqk + dT1 + dQs +
           dW + dKb + dgam + dbu;
  }
};

// State columns per pass CTA: 32 while the 2 x (B H) x (d_v / 32) CTAs fit
// in one wave of the 148 SMs, else 64 (fewer CTAs reading the same operands).
int pass_width(int BH, int dv) { return (size_t)2 * BH * (dv / 32) <= 148 ? 32 : 64; }

// The first kernel of a call launches plainly (it follows arbitrary work on
// the stream); the others as programmatic dependents of the one before.
template <typename Kern>
cudaError_t launch_k(Kern kern, dim3 grid, size_t smem, const ChunkBwdArgs& a, cudaStream_t stream,
                     int nth = kThreads, bool dependent = true) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(nth);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = dependent ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

// dO [B, T, H, d_v] bf16 as a 4-D tensor map (channel, head, token, batch),
// box 64 channels x 64 tokens, 128-byte swizzle; tokens past T read as zeros.
PFN_cuTensorMapEncodeTiled_v12000 bwd_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}
bool bwd_map_bf16(CUtensorMap* map, const void* base, int B, int T, int H, int d) {
  auto enc = bwd_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor-core state passes (bf16, d_k = d_v = 128): one CTA per
// (sequence, head) of the group and role, a programmatic dependent of the
// preparation kernel.
cudaError_t launch_pass_tc(const ChunkBwdArgs& a, int BH, int B, WorkspaceHeader* hdr, cudaStream_t stream) {
  CUtensorMap mo;
  if (!bwd_map_bf16(&mo, a.d_o, B, a.T, a.H, 128)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(tcpass::bwd_pass_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)tcpass::kSmem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)BH, 2);
  cfg.blockDim = dim3(tcpass::kThreads);
  cfg.dynamicSmemBytes = tcpass::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, tcpass::bwd_pass_tc_kernel, mo, a, hdr);
}

// The tensor-core passes run one CTA per (sequence, head) and role, with all
// 128 value channels in one tensor-memory accumulator; the warp-level passes
// split the value channels over 4 CTAs, which keeps more SMs busy when the
// chains are few.  The tensor-core path also takes its operands from the
// forward's preparation kernel (four tiles per SM) instead of the one-tile-
// per-SM preparation of the warp-level path.  Measured per call: 466 vs 493
// us at B1 H16 T4096 and 10.1 vs 12.2 ms at B8 H32 T8192 in favour of the
// tensor-core path; it is taken from 16 (sequence, head) chains on.
bool tc_pass_pays(int BH) { return BH >= 16; }

template <typename IO, int DK, int DV>
cudaError_t launch_chunk_typed(const ChunkBwdArgs& a_in, int BH, int B, WorkspaceHeader* hdr, cudaStream_t stream) {
  ChunkBwdArgs a = a_in;
  a.tc_rec = !std::is_same<IO, float>::value && kTcPass<DK, DV> && tc_pass_pays(BH);
  const dim3 grid((unsigned)a.NC * BH);  // chunk-major within each (sequence, head)
  cudaError_t e;
  if (std::is_same<IO, float>::value) {
    e = launch_k(bwd_prep_kernel<float, DK, DV>, grid, prep_smem<DK, DV>(), a, stream, kThreads, false);
  } else if (a.tc_rec) {
    // the forward's preparation kernel (tcgen05, four tiles per SM) in its
    // backward mode writes the same operands in the same layouts
    const PrepBwdOut out{reinterpret_cast<uint8_t*>(a.prec), (size_t)PassRec<DK>::n * 2, a.Pkk,
                         reinterpret_cast<bf16*>(a.Tm), a.U, a.gam, a.bh0, BH};
    e = launch_prep_for_backward(static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k),
                                 static_cast<const bf16*>(a.v), static_cast<const bf16*>(a.g),
                                 static_cast<const bf16*>(a.beta), a.scale, B, a.T, a.H, a.gate, out, hdr, stream);
  } else {
    e = launch_k(bwd_prep_bf16_kernel<DK, DV>, grid, PrepPlanB<DK, DV>::bytes, a, stream, kThreads, false);
  }
  if (e != cudaSuccess) return e;
  const bool w32 = pass_width(BH, DV) == 32;
  if constexpr (std::is_same<IO, float>::value) {
    if (w32)
      e = launch_k(bwd_pass_kernel<IO, DK, DV, 32>, dim3(BH * (DV / 32), 2), pass_smem<DK, DV, 32>(), a, stream,
                   kPassThreads);
    else
      e = launch_k(bwd_pass_kernel<IO, DK, DV, 64>, dim3(BH * (DV / 64), 2), pass_smem<DK, DV, 64>(), a, stream,
                   kPassThreads);
  } else if (a.tc_rec) {
    e = launch_pass_tc(a, BH, B, hdr, stream);
  } else {
    (void)hdr;
    if (w32)
      e = launch_k(bwd_pass_bf16_kernel<DK, DV, 32>, dim3(BH * (DV / 32), 2), pass_bf16_smem<DK, DV, 32>(), a,
                   stream, kPassThreads);
    else
      e = launch_k(bwd_pass_bf16_kernel<DK, DV, 64>, dim3(BH * (DV / 64), 2), pass_bf16_smem<DK, DV, 64>(), a,
                   stream, kPassThreads);
  }
  if (e != cudaSuccess) return e;
  if constexpr (std::is_same<IO, float>::value)
    e = launch_k(bwd_local_a_kernel<IO, DK, DV>, grid, local_a_smem<DK, DV>(), a, stream);
  else
    e = launch_k(bwd_local_a_bf16_kernel<DK, DV>, grid, LocalAPlanB<DK, DV>::bytes, a, stream, kLaThreads);
  if (e != cudaSuccess) return e;
  if constexpr (std::is_same<IO, float>::value)
    return launch_k(bwd_local_b_kernel<IO, DK, DV>, grid, local_b_smem<DK, DV>(), a, stream);
  else
    return launch_k(bwd_local_b_bf16_kernel<DK, DV>, grid, LocalBPlanB<DK, DV>::bytes, a, stream);
}

template <typename IO>
cudaError_t launch_chunk_dims(const ChunkBwdArgs& a, int BH, int B, WorkspaceHeader* hdr, int dk, int dv,
                              cudaStream_t stream) {
  if (dk == 128 && dv == 128) return launch_chunk_typed<IO, 128, 128>(a, BH, B, hdr, stream);
  if (dk == 128 && dv == 64) return launch_chunk_typed<IO, 128, 64>(a, BH, B, hdr, stream);
  if (dk == 64 && dv == 128) return launch_chunk_typed<IO, 64, 128>(a, BH, B, hdr, stream);
  return launch_chunk_typed<IO, 64, 64>(a, BH, B, hdr, stream);
}

static_assert(LocalBPlanB<128, 128>::bytes <= 232448 && PrepPlanB<128, 128>::bytes <= 232448, "shared memory per CTA");
static_assert(prep_smem<128, 128>() <= 232448 && local_a_smem<128, 128>() <= 232448 &&
                  local_b_smem<128, 128>() <= 232448 && pass_smem<128, 128, 64>() <= 232448,
              "shared memory per CTA");

}  // namespace

// The workspace starts with a WorkspaceHeader (the error word of the bounded
// waits of the tensor-core passes), then the per-chunk records.
size_t backward_workspace_bytes(int B, int T, int H, int dk, int dv, int dtype) {
  const size_t nrec = (size_t)B * H * (((size_t)T + kC - 1) / kC);
  return sizeof(WorkspaceHeader) + nrec * WsPlan(dk, dv, dtype == KDA_F32).per_rec() * sizeof(float);
}

cudaError_t launch_backward(const void* q, const void* k, const void* v, const void* g, const void* beta,
                            float scale, const float* s0, const void* d_o, const float* dsT, void* dq, void* dk_out,
                            void* dv_out, void* dg, void* dbeta, float* ds0, int B, int T, int H, int dk, int dv,
                            int dtype, int gate, void* ws, size_t ws_bytes, cudaStream_t stream, float* dq32,
                            float* dk32, WorkspaceHeader* hdr) {
  if (!hdr) {  // the header leads the caller's workspace
    if (ws_bytes < sizeof(WorkspaceHeader)) return cudaErrorInvalidValue;
    hdr = static_cast<WorkspaceHeader*>(ws);
    ws = static_cast<uint8_t*>(ws) + sizeof(WorkspaceHeader);
    ws_bytes -= sizeof(WorkspaceHeader);
  }
  {
    const cudaError_t e0 = cudaMemsetAsync(hdr, 0, sizeof(WorkspaceHeader), stream);
    if (e0 != cudaSuccess) return e0;
  }
  ChunkBwdArgs a;
  a.tc_rec = 0;
  a.dq32 = dq32, a.dk32 = dk32;
  a.q = q, a.k = k, a.v = v, a.g = g, a.beta = beta, a.d_o = d_o;
  a.s0 = s0, a.dsT = dsT;
  a.dq = dq, a.dk = dk_out, a.dv = dv_out, a.dg = dg, a.dbeta = dbeta, a.ds0 = ds0;
  a.scale = scale, a.T = T, a.H = H, a.NC = (T + kC - 1) / kC, a.gate = gate;
  // (sequence, head) pairs per launch group: as many as the workspace holds
  const int BH = B * H;
  const size_t per_bh = backward_workspace_bytes(1, T, 1, dk, dv, dtype) - sizeof(WorkspaceHeader);
  const int nfit = (int)std::min<size_t>((size_t)BH, ws_bytes / per_bh);
  if (nfit < 1) return cudaErrorInvalidValue;
  const WsPlan p(dk, dv, dtype == KDA_F32);
  for (int bh0 = 0; bh0 < BH; bh0 += nfit) {
    const int nbh = std::min(nfit, BH - bh0);
    const size_t nrec = (size_t)nbh * a.NC;
    float* w = static_cast<float*>(ws);
    auto take = [&](size_t per) {
      float* r = w;
      w += nrec * per;
      return r;
    };
    a.bh0 = bh0;
    a.W = take(p.W), a.U = take(p.U), a.Qp = take(p.Qp), a.Kb = take(p.Kb);
    a.Wt = take(p.Wt), a.Qpt = take(p.Qpt), a.Kbt = take(p.Kbt);
    a.Aqk = take(p.Aqk), a.prec = reinterpret_cast<bf16*>(take(p.prec));
    a.Tm = take(p.Tm), a.Pkk = take(p.Pkk), a.gam = take(p.gam);
    a.S0c = take(p.S0c), a.dSc = take(p.dSc), a.Vp = take(p.Vp), a.dVp = take(p.dVp);
    a.dAqk = take(p.dAqk), a.dT1 = take(p.dT1), a.dQs = take(p.dQs), a.dW = take(p.dW), a.dKb = take(p.dKb);
    a.dgam = take(p.dgam), a.dbu = take(p.dbu);
    const cudaError_t e = dtype == KDA_F32 ? launch_chunk_dims<float>(a, nbh, B, hdr, dk, dv, stream)
                                           : launch_chunk_dims<__nv_bfloat16>(a, nbh, B, hdr, dk, dv, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace kda
