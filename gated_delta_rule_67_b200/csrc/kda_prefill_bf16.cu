// kda_prefill_bf16.cu -- bf16 chunked KDA prefill on the sm_100a tensor cores.
//
// Chunkwise form of the KDA recurrence (KimiLinear article: section 2.3 for
// the update, section 3.1 for the chunked evaluation, section 3.2 for the
// C x C per-chunk score matrix).  Per chunk of C = 64 tokens, with the
// in-chunk inclusive cumulative log-gate G_i (per key channel), S0 the state
// entering the chunk and the rows of K, Q, V the chunk's tokens:
//
//   A_kk[i,j] = beta_i (k_i*exp(G_i - G_r)) . (k_j*exp(G_r - G_j))   j <  i
//   A_qk[i,j] = scale (q_i*exp(G_i - G_r)) . (k_j*exp(G_r - G_j))    j <= i
//   T  = (I + A_kk)^-1                                  (unit lower triangular)
//   W  = T diag(beta) K+,   K+_i = k_i*exp(G_i)          (decayed from chunk start)
//   U  = T diag(beta) V
//   V' = U - W S0                                        (the chunk's effective writes)
//   O  = Q+ S0 + A_qk V',   Q+_i = scale q_i*exp(G_i)
//   S  = Diag(exp(G_C)) S0 + Kbar^T V',   Kbar_j = k_j*exp(G_C - G_j)
//
// (derived from the token recurrence: S_t = Diag(a_t) S_{t-1} + k_t u_t^T
// with u_t = beta_t (v_t - S_{t-1}^T (a_t*k_t)); collecting the u_t of one
// chunk gives the unit-triangular system (I + A_kk) U' = beta*(V - K+ S0)).
// G_r is a reference point inside the chunk (token 31): the products are
// independent of it, and centring keeps both exponential factors near 1.
//
// Kernels:
//  1. kda_chunk_prep: one CTA per (sequence, head, chunk), fully parallel,
//     four CTAs per SM.  TMA brings q, k, v, g (64 x 128 bf16 tiles, 128-byte
//     swizzle); the CTA computes G and the decayed operands, the two score
//     matrices with one tcgen05 MMA (M=128: rows 0-63 give A_kk, rows 64-127
//     give A_qk), the triangular inverse in fp32 by 16 x 16 blocks (diagonal
//     blocks by forward substitution, the others with warp-level tf32
//     products), and W^T, U^T with two more MMAs.  It writes, per chunk, a
//     record of ready-to-use operand images (already in the swizzled
//     shared-memory layout the MMAs read): -W^T (128 key-channel rows x 64
//     tokens), Q+ (64 token rows x 128), A_qk (64 x 64), Kbar (64 x 128),
//     U^T (128 x 64) and gamma = exp(G_C) (128 fp32).  In its backward mode
//     it writes the backward's per-chunk operands instead.
//  2. kda_state_pass: walks chunks in order with the state S^T (d_v x d_k,
//     fp32) resident in tensor memory.  Per chunk: S0^T -> bf16 operand;
//     P = S0^T (-W)^T; V'^T = U^T + P while S^T is decayed by gamma and
//     O^T = S0^T Q+^T is formed; then O^T += V'^T A_qk^T and S^T += V'^T Kbar.
//     The next chunk's record is prefetched with bulk copies while the
//     current one is processed.  One CTA per (sequence, head), or, when few
//     chains cover many chunks, the chunk-parallel scan: one CTA per group
//     of chunks and pass (phase 1: offsets and transitions; phase 3: the
//     outputs from each group's true start state).
//  3. kda_scan_combine_kernel: chains the groups' affine state maps of the
//     scan on the tensor cores (one CTA per chain).
//
// Everything is transposed relative to the token-major notation above so
// that every MMA has M = 128 (the d_v or d_k dimension) and each TMEM lane is
// one channel.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>

#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int kC = 64;    // chunk length
constexpr int kD = 128;   // d_k = d_v
constexpr int kRefTok = 31;  // reference token of the factored form: the end of the second 16-token stride
static_assert(kRefTok == 2 * 16 - 1, "pass 1 takes G_r as the sum of the first two stride totals");

// --- per-chunk record in the workspace (byte offsets) -----------------------
constexpr uint32_t kRecW = 0;           // -W^T: 128 key-channel rows x 64 tokens (MN-major B of P; 16 KiB)
constexpr uint32_t kRecQ = 16384;       // Q+: 64 token rows x 128 channels (K-major B of O^T = S0^T Q+^T; 16 KiB)
constexpr uint32_t kRecAqk = 32768;     // A_qk: 64 rows i x 64 columns j (K-major B of O^T += V'^T A_qk^T; 8 KiB)
constexpr uint32_t kRecKbar = 40960;    // Kbar: token-row tile 64 x 128 (16 KiB)
constexpr uint32_t kRecU = 57344;       // U^T: K-major, 128 rows (channel) x 64 (token) (16 KiB)
constexpr uint32_t kRecGamma = 73728;   // gamma: 128 fp32
constexpr uint32_t kRecBytes = 74240;

// --- prep kernel: shared memory (byte offsets from a 1024-aligned base) ---
// 52 KiB, so that four CTAs share an SM.
// Region A (32 KiB) is a 128-row K-major tile in two 64-channel halves of
// 16 KiB.  Rows 0-63 of each half ([0,8K) and [16K,24K)) first hold g, then
// K+_r, which stays for the W product and is finally overwritten by the -W
// staging tile; rows 64-127 ([8K,16K) and [24K,32K)) hold q, then Q+_r.
// Once the score MMA is done, the v tile takes [8K,16K) and [24K,32K) (a
// 64-row tile whose channel halves lie 16 KiB apart); its second half comes
// after the A_qk staging tile at [24K,32K) has been bulk-stored.
// Region B (16 KiB): the k tile, turned in place into K-_r (score B operand);
// then the 10 A_kk blocks [0,10K) and six T blocks [10K,16K); after the
// solve the (T diag beta)^T operand [0,8K); finally the U^T staging tile.
// Region T (4 KiB): the last four T blocks.
constexpr uint32_t kP1A = 0;
constexpr uint32_t kP1B = 32768;
constexpr uint32_t kP1T = 49152;
constexpr uint32_t kP1Bytes = 53248;
constexpr uint32_t kP1V = kP1A + 8192;       // v tile (half stride 16 KiB), after the score MMA
constexpr uint32_t kP1B2 = kP1B;             // (T diag beta)^T, K-major 64 x 64, after the solve
constexpr uint32_t kP1QT = kP1A + 24576;     // A_qk staging (bulk-stored before v's second half lands)
constexpr int kP1Threads = 256;
constexpr int kP1Blocks = 4;                 // CTAs per SM: 4 x 128 TMEM columns, 4 x ~55 KiB shared memory
// Per-chunk safe range of the factored form: every channel's cumulative
// log-gate over the chunk must stay above -kSafeSpan, so that each factor
// exp(+-(G_i - G_r)), exp(G_r), exp(G_C - G_r) lies in [e^-64, e^64].
constexpr float kSafeSpan = 64.f;

// --- state-pass kernel shared memory --------------------------------------
constexpr uint32_t kStage = 74752;      // record rounded up to 1024
constexpr uint32_t kP2Out = 2 * kStage;     // two 16 KiB output staging tiles [half][token][64 ch] bf16
constexpr uint32_t kP2Bytes = kP2Out + 2 * 16384;

constexpr uint32_t kWaitLimit = 1u << 24;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ void stbf(uint8_t* base, uint32_t off, float x) {
  *reinterpret_cast<bf16*>(base + off) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 t = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&t);
}
// 8 consecutive K elements (k0 % 8 == 0) of row r of a K-major tile: one 16-byte store.
__device__ __forceinline__ void st_kmajor8(uint8_t* tile, uint32_t r, uint32_t k0, uint32_t rows, const float* v) {
  uint4 w = make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]), pack2(v[6], v[7]));
  *reinterpret_cast<uint4*>(tile + kmajor_off(r, k0, rows)) = w;
}

__device__ __forceinline__ void wait_or_flag(uint64_t* bar, uint32_t parity, WorkspaceHeader* hdr, uint32_t where) {
  if (!mbar_wait(bar, parity, kWaitLimit)) {
    atomicOr(&hdr->error, 1u);
    atomicExch(&hdr->where, where);
  }
}

// =============================================================== kernel 1
__device__ __forceinline__ float2 ld_bf2(const uint8_t* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
// 8 bf16 (16 bytes, 16-byte aligned) <-> 8 floats.
__device__ __forceinline__ void ld8(const uint8_t* p, float* f) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u[e]));
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}
__device__ __forceinline__ void st8(uint8_t* p, const float* f) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}
// The lower-triangular 64 x 64 matrices A_kk and T are kept as 16 x 16 fp32
// blocks (I, J), J <= I, numbered p = I(I+1)/2 + J; A blocks in region B,
// T blocks 0-5 after them in region B and T blocks 6-9 in region T.
__device__ __forceinline__ int blk(int I, int J) { return I * (I + 1) / 2 + J; }
// Element (r, c) of a 16 x 16 block: rows of 16 floats with the float4 column
// XOR-ed by (r/2)%4, so that 8 consecutive rows at one float4 column hit 8
// different 16-byte bank groups.
__device__ __forceinline__ int bidx(int r, int c) { return r * 16 + ((((c >> 2) ^ ((r >> 1) & 3)) << 2) | (c & 3)); }
__device__ __forceinline__ float* a_blk(uint8_t* sm, int p) { return reinterpret_cast<float*>(sm + kP1B) + p * 256; }
__device__ __forceinline__ float* t_blk(uint8_t* sm, int p) {
  return p < 6 ? reinterpret_cast<float*>(sm + kP1B + 10240) + p * 256
               : reinterpret_cast<float*>(sm + kP1T) + (p - 6) * 256;
}
// Warp-level 16x16x16 product acc += P Q of row-major fp32 16x16 blocks, with
// mma.sync m16n8k8 (tf32 operands rounded to nearest).  acc[nh] holds the
// 16x8 accumulator fragment of columns 8nh..8nh+7: rows g and g+8, columns
// 2t and 2t+1, where g = lane / 4 and t = lane % 4.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void block_mma_tf32(float (&acc)[2][4], const float* P, const float* Q, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int kh = 0; kh < 2; ++kh) {
    const uint32_t a0 = to_tf32(P[bidx(g, 8 * kh + t)]), a1 = to_tf32(P[bidx(g + 8, 8 * kh + t)]);
    const uint32_t a2 = to_tf32(P[bidx(g, 8 * kh + t + 4)]), a3 = to_tf32(P[bidx(g + 8, 8 * kh + t + 4)]);
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
      const uint32_t b0 = to_tf32(Q[bidx(8 * kh + t, 8 * nh + g)]), b1 = to_tf32(Q[bidx(8 * kh + t + 4, 8 * nh + g)]);
      asm volatile(
          "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
          "{%0,%1,%2,%3};"
          : "+f"(acc[nh][0]), "+f"(acc[nh][1]), "+f"(acc[nh][2]), "+f"(acc[nh][3])
          : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
  }
}
__device__ __forceinline__ void store_block_frag(float* X, const float (&acc)[2][4], int lane, float sign) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nh = 0; nh < 2; ++nh) {
    X[bidx(g, 8 * nh + 2 * t)] = sign * acc[nh][0];
    X[bidx(g, 8 * nh + 2 * t + 1)] = sign * acc[nh][1];
    X[bidx(g + 8, 8 * nh + 2 * t)] = sign * acc[nh][2];
    X[bidx(g + 8, 8 * nh + 2 * t + 1)] = sign * acc[nh][3];
  }
}

// kScalarGate: the forget gate is one log-gate per (token, head) read from
// g_head (Gated DeltaNet), or none when g_head is null (DeltaNet); otherwise
// the per-channel g tile comes in by TMA (KDA).  kPrep: the inputs are raw
// and `prep` (kda_prep bits) says which ones to prepare here: q, k scaled to
// unit length per token (the per-token factors are applied wherever q and k
// are read), log-sigmoid of g, sigmoid of beta.  kBwd: the operands go to the
// backward instead (`bo`: W, Q+, Kbar, A_qk as token-row tiles, P and U in
// fp32, T in bf16, gamma) for the (sequence, head) pairs bo.bh0 onwards; the
// forward record is not written.
template <bool kScalarGate, bool kPrep, bool kBwd = false>
__global__ void __launch_bounds__(kP1Threads, kP1Blocks)
    kda_chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                          const bf16* __restrict__ beta, float scale, uint8_t* __restrict__ records,
                          WorkspaceHeader* hdr, int T, int H, int NC, const bf16* __restrict__ g_head, int prep,
                          const PrepBwdOut bo) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ uint64_t bar_in, bar_v, bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ float sbeta[kC];
  __shared__ float sgh[kScalarGate ? kC : 1];  // per-head log-gates of the chunk (zeros without a gate)
  __shared__ float snq[kPrep ? kC : 1], snk[kPrep ? kC : 1];  // per-token sums of q^2, k^2 (fused L2 norm)
  __shared__ __align__(16) float segr[kD];  // per channel: exp(G_r) (factored form) or 1 (exact path); scales W in its extraction
  const bool l2n = kPrep && (prep & KDA_PREP_L2NORM_QK);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x % NC;
  const int bh = (kBwd ? bo.bh0 : 0) + (int)(blockIdx.x / NC);
  const int h = bh % H, b = bh / H;
  const int t0 = chunk * kC;
  const int L = min(kC, T - t0);
  // the record of this chunk and the offsets of its images in it
  const size_t ri = blockIdx.x;  // backward: the index of its per-chunk arrays too
  uint8_t* rec = kBwd ? bo.rec + ri * bo.rec_stride : records + ri * kRecBytes;
  constexpr uint32_t oRecQ = kBwd ? kTcRecQp : kRecQ, oRecKbar = kBwd ? kTcRecKb : kRecKbar;
  constexpr uint32_t oRecAqk = kBwd ? kTcRecAqk : kRecAqk;

  if (tid == 0) {
    mbar_init(&bar_in, 1);
    mbar_init(&bar_v, 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
    mbar_expect_tx(&bar_in, (kScalarGate ? 2 : 3) * 16384);
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      if (!kScalarGate) tma_load_4d(sm + kP1A + kb * 16384, &tm_g, &bar_in, kb * 64, h, t0, b);  // rows 0-63
      tma_load_4d(sm + kP1A + kb * 16384 + 8192, &tm_q, &bar_in, kb * 64, h, t0, b);     // rows 64-127
      tma_load_4d(sm + kP1B + kb * 8192, &tm_k, &bar_in, kb * 64, h, t0, b);
    }
  }
  if (warp == 0) tmem_alloc(&tmem_base, 128);
  // beta is a strided gather (one 2-byte value per token): read it now, park
  // it in shared memory only after the gate scan, off the first barrier's path
  const float beta_x = (tid < L) ? __bfloat162float(beta[((size_t)b * T + t0 + tid) * H + h]) : 0.f;
  if (kScalarGate && tid >= kC && tid < 2 * kC) {
    const int i = tid - kC;
    const float x = (g_head && i < L) ? __bfloat162float(g_head[((size_t)b * T + t0 + i) * H + h]) : 0.f;
    sgh[i] = (kPrep && g_head && i < L) ? prep_gate(prep, x) : x;
  }
  if (kPrep && tid >= 2 * kC && tid < 3 * kC) {
    snq[tid - 2 * kC] = 0.f;
    snk[tid - 2 * kC] = 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The state pass may now be scheduled: it waits for this grid to finish
  // before it reads anything, and this CTA already holds its tensor memory.
  grid_dep_launch();
  const uint32_t tm = tmem_base;
  wait_or_flag(&bar_in, 0, hdr, 1);

  // Thread = (8-channel group cg, token lane tg) in the shuffle-scan form of
  // pass 1 and the passes after it; thread = (token mi, 16 channels of each
  // 64-channel half at 16 q4) in the tensor-core form (per-channel gates given
  // as bf16 log-gates, the KDA case), whose G comes from one product.
  constexpr bool kMmaScan = !kScalarGate && !kPrep;
  const int cg = 2 * warp + (lane >> 4);
  const int tg = lane & 15;
  const int c8 = 8 * cg;
  const int mi = 32 * (warp & 1) + lane;
  const int q4 = 2 * ((warp >> 1) & 1) + (warp >> 2);
  const uint32_t lane_tm = tm + ((uint32_t)((warp & 3) * 32) << 16);
  // shuffle-scan form: G parked at columns (warp / 4) * 32 + 8t + e of this lane
  const uint32_t g_tm = lane_tm + (warp >> 2) * 32;
  // tensor-core form: accumulator [0,64), the ones operand [64,96), the parked first half [96,128)
  constexpr uint32_t kTmL = 64, kTmG0 = 96;
  float* sgref = reinterpret_cast<float*>(sm + kP1T);  // region T, idle until the solve:
  float* sgend = sgref + kD;                            // G at tokens 31 and 63, exp(G_C - G_r)
  float* segb = sgref + 2 * kD;
  float gref[8], gend[8];
  int slow;
  if constexpr (kMmaScan) {
    // ---- pass 1 (tensor cores): G = L g with L the 64 x 64 lower-triangular
    // matrix of ones as the A operand in tensor memory (rows 64-127 repeat
    // rows 0-63, so that the lanes of every warp hold tokens) and the g tile
    // as the MN-major B operand, one 64-channel half at a time.  The products
    // are exact (g is bf16, L is 0 or 1) and the sums fp32.
    if (warp < 4) {
      uint32_t lw[32];
#pragma unroll
      for (int e = 0; e < 32; ++e)
        lw[e] = (2 * e <= mi ? 0x3F80u : 0u) | (2 * e + 1 <= mi ? 0x3F800000u : 0u);  // bf16 1.0 pairs
      tmem_st32u(lane_tm + kTmL, lw);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {
      if (tid == 0) {
        const uint32_t idesc = idesc_bf16_f32(128, 64, 0, 1);
        const uint64_t b0 = desc_sw128(smem_u32(sm + kP1A + hf * 16384), 16384, 1024);
#pragma unroll
        for (int k = 0; k < kC / 16; ++k)
          mma_bf16_ts(tm, tm + kTmL + k * 8, b0 + (uint64_t)((k * 2048) >> 4), idesc, k > 0);
        mma_commit(&bar_mma);
      }
      wait_or_flag(&bar_mma, hf, hdr, 5 + hf);
      tc_fence_after();
      float Gq[16];
      tmem_ld16(lane_tm + 16 * q4, Gq);
      if (lane == 31) {  // tokens 31 (the reference) and 63 (the chunk end)
        float4* dst = reinterpret_cast<float4*>(((warp & 1) ? sgend : sgref) + 64 * hf + 16 * q4);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_float4(Gq[4 * e], Gq[4 * e + 1], Gq[4 * e + 2], Gq[4 * e + 3]);
      }
      if (hf == 0) {  // the first half waits in this lane's spare columns; the accumulator takes the second
        tmem_st16(lane_tm + kTmG0 + 16 * (warp >> 2), Gq);
        tmem_wait_st();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
      }
    }
    __syncthreads();  // G at tokens 31 and 63 is in shared memory
    if (tid < kC) sbeta[tid] = beta_x;
    bool unsafe = false;
    if (tid < kD) {
      const float gr = sgref[tid], ge = sgend[tid];
      unsafe = ge < -kSafeSpan;
      segr[tid] = __expf(gr);
      segb[tid] = __expf(ge - gr);
      (kBwd ? bo.gam + ri * kD : reinterpret_cast<float*>(rec + kRecGamma))[tid] = expf(ge);
    }
    slow = __syncthreads_or(unsafe);  // the g tile is dead from here on
  } else {
    // ---- pass 1: in-chunk cumulative log-gate.  Thread = (8-channel group cg,
    // token lane tg) owning tokens tg, tg+16, tg+32, tg+48: the 8 lanes of a
    // quarter-warp then touch rows of 8 different swizzle phases (no bank
    // conflicts).  Inclusive scans over the 16 lanes of each token stride,
    // then the stride totals are added in order.
    float G[4][8];
    if (l2n) {  // per-token sums of squares of q and k over the 128 channels
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int i = tg + 16 * t;
        float q8[8], k8[8];
        ld8(sm + kP1A + kmajor_off(kC + i, c8, 128), q8);
        ld8(sm + kP1B + kmajor_off(i, c8, kC), k8);
        float sq2 = 0.f, sk2 = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          sq2 = fmaf(q8[e], q8[e], sq2);
          sk2 = fmaf(k8[e], k8[e], sk2);
        }
        atomicAdd(&snq[i], sq2);
        atomicAdd(&snk[i], sk2);
      }
    }
    if (!kScalarGate) {
#pragma unroll
      for (int t = 0; t < 4; ++t) ld8(sm + kP1A + kmajor_off(tg + 16 * t, c8, 128), G[t]);
      if (kPrep && (prep & KDA_PREP_GATE_LOGSIGMOID)) {
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int e = 0; e < 8; ++e) G[t][e] = tg + 16 * t < L ? log_sigmoid_fast(G[t][e]) : 0.f;  // padding: no decay
      }
    } else {  // one log-gate per token for every channel (zero without a gate)
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int e = 0; e < 8; ++e) G[t][e] = sgh[tg + 16 * t];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float tot[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        float x = G[t][e];
#pragma unroll
        for (int d = 1; d < 16; d <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, d, 16);
          if (tg >= d) x += y;
        }
        G[t][e] = x;
        tot[t] = __shfl_sync(0xffffffffu, x, 15, 16);
      }
      G[1][e] += tot[0];
      G[2][e] += tot[0] + tot[1];
      G[3][e] += (tot[0] + tot[1]) + tot[2];
      gref[e] = tot[0] + tot[1];                 // G at token 31
      gend[e] = ((tot[0] + tot[1]) + tot[2]) + tot[3];  // G at token 63 (= G_C; padding has g = 0)
    }
    // G goes to tensor memory until the decayed operands are formed (held in
    // registers across that stretch it would spill to local memory): thread
    // (warp, lane) keeps its 32 values in its own lane (warp % 4) * 32 + lane,
    // columns (warp / 4) * 32 + 8t + e.  The score MMA overwrites them later.
    tmem_st32(g_tm, &G[0][0]);
    tmem_wait_st();
    if (tid < kC) sbeta[tid] = (kPrep && tid < L) ? prep_beta(prep, beta_x) : beta_x;
    bool unsafe = false;
#pragma unroll
    for (int e = 0; e < 8; ++e) unsafe |= gend[e] < -kSafeSpan;
    if (tg == 0) {
      float* gam = (kBwd ? bo.gam + ri * kD : reinterpret_cast<float*>(rec + kRecGamma)) + c8;
      *reinterpret_cast<float4*>(gam) = make_float4(expf(gend[0]), expf(gend[1]), expf(gend[2]), expf(gend[3]));
      *reinterpret_cast<float4*>(gam + 4) = make_float4(expf(gend[4]), expf(gend[5]), expf(gend[6]), expf(gend[7]));
    }
    slow = __syncthreads_or(unsafe);  // the g tile is dead from here on

  }

  if (!slow) {
    if constexpr (kMmaScan) {
      // ---- pass 2 (factored form), token mi and four 8-channel pieces: the
      // decayed operands relative to token kRefTok.  Each (token, piece) slot
      // of the k, q and g tiles belongs to one thread, read before it is
      // overwritten; the per-channel factors come from shared memory.
#pragma unroll 1
      for (int p = 0; p < 4; ++p) {
        const int hf = p >> 1, c = 64 * hf + 16 * q4 + 8 * (p & 1);
        float Gt[8], f8[8], k8[8], q8[8], w[8], ex[8];
        tmem_ld8(hf == 0 ? lane_tm + kTmG0 + 16 * (warp >> 2) + 8 * (p & 1) : lane_tm + 16 * q4 + 8 * (p & 1), Gt);
        const uint32_t oK = kmajor_off(mi, c, kC);        // 64-row tiles: k, K-_r, Kbar, the Q+ image
        const uint32_t oA = kmajor_off(mi, c, 128);       // row mi of region A
        const uint32_t oQ = kmajor_off(kC + mi, c, 128);  // row 64+mi of region A (q, then Q+_r)
        ld8(sm + kP1B + oK, k8);
        ld8(sm + kP1A + oQ, q8);
        auto ld8f = [](const float* src, float* f) {  // 8 per-channel factors, two 16-byte loads
          const float4 a0 = *reinterpret_cast<const float4*>(src), a1 = *reinterpret_cast<const float4*>(src + 4);
          f[0] = a0.x, f[1] = a0.y, f[2] = a0.z, f[3] = a0.w, f[4] = a1.x, f[5] = a1.y, f[6] = a1.z, f[7] = a1.w;
        };
        ld8f(sgref + c, f8);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          Gt[e] -= f8[e];  // G - G_r
          ex[e] = __expf(Gt[e]);
          q8[e] *= scale;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = k8[e] * ex[e];
        st8(sm + kP1A + oA, w);               // K+_r (over the dead g rows)
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = q8[e] * ex[e];
        st8(sm + kP1A + oQ, w);               // Q+_r (in place of q)
        ld8f(segr + c, f8);
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = q8[e] * (ex[e] * f8[e]);
        st8(rec + oRecQ + oK, w);             // Q+ image
#pragma unroll
        for (int e = 0; e < 8; ++e) ex[e] = __expf(-Gt[e]);
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = k8[e] * ex[e];
        st8(sm + kP1B + oK, w);               // K-_r, in place of k
        ld8f(segb + c, f8);
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = k8[e] * (ex[e] * f8[e]);
        st8(rec + oRecKbar + oK, w);          // Kbar image = k exp(G_C - G_i)
      }
    } else {
      // ---- pass 2 (factored form): decayed operands relative to token kRefTok
      float egr[8], egb[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        egr[e] = __expf(gref[e]);
        egb[e] = __expf(gend[e] - gref[e]);
      }
      if (tg == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) segr[c8 + e] = egr[e];
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int i = tg + 16 * t;
        const uint32_t oK = kmajor_off(i, c8, kC);        // 64-row tiles: k, K-_r, Kbar
        const uint32_t oA = kmajor_off(i, c8, 128);       // row i of region A
        const uint32_t oQ = kmajor_off(kC + i, c8, 128);  // row 64+i of region A (q, then Q+_r)
        float k8[8], q8[8], Gt[8];
        tmem_ld8(g_tm + 8 * t, Gt);
        ld8(sm + kP1B + oK, k8);
        ld8(sm + kP1A + oQ, q8);
        if (l2n) {
          const float rk = rsqrtf(snk[i] + kL2Eps), rq = rsqrtf(snq[i] + kL2Eps);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            k8[e] *= rk;
            q8[e] *= rq;
          }
        }
        // the start-decayed operands first, then the end-decayed ones, so that
        // fewer values are live at once (64 registers at 4 CTAs per SM)
        float w[8];
        {
          float ex[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            ex[e] = __expf(Gt[e] - gref[e]);
            q8[e] *= scale;
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = k8[e] * ex[e];
          st8(sm + kP1A + oA, w);               // K+_r (over the dead g rows)
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = q8[e] * ex[e];
          st8(sm + kP1A + oQ, w);               // Q+_r (in place of q)
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = q8[e] * (ex[e] * egr[e]);
          st8(rec + oRecQ + oK, w);             // Q+ image (64 token rows, the layout of the k tile)
        }
        {
          float ei[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) ei[e] = __expf(gref[e] - Gt[e]);
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = k8[e] * ei[e];
          st8(sm + kP1B + oK, w);               // K-_r, in place of k
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = k8[e] * (ei[e] * egb[e]);
          st8(rec + oRecKbar + oK, w);          // Kbar image = k exp(G_C - G_i)
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- score MMA: D[0:128, 0:64] = [K+_r ; Q+_r] (128 x 128) . K-_r^T
    if (tid == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
      const uint64_t a0 = desc_sw128(smem_u32(sm + kP1A), 16, 1024), b0 = desc_sw128(smem_u32(sm + kP1B), 16, 1024);
#pragma unroll
      for (int k = 0; k < kD / 16; ++k)
        mma_bf16(tm, a0 + (uint64_t)(((k / 4) * 16384 + (k % 4) * 32) >> 4),
                 b0 + (uint64_t)(((k / 4) * 8192 + (k % 4) * 32) >> 4), idesc, k > 0);
      mma_commit(&bar_mma);
    }
    wait_or_flag(&bar_mma, 0, hdr, 2);
    tc_fence_after();

    // ---- rows 0-63 -> A_kk blocks (times beta_i, strictly lower); rows 64-127 -> A_qk staging
    {
      const int row = (warp & 3) * 32 + lane;
      const int col0 = (warp >> 2) * 32;
      float v[32];
      tmem_ld32(tm + ((uint32_t)((warp & 3) * 32) << 16) + col0, v);
      if (row < kC) {
        const int i = row, I = i >> 4;
        const float bi = sbeta[i];
        if (kBwd) {  // P row i, columns col0 .. col0 + 31 (zero on and above the diagonal)
          float4* Pr = reinterpret_cast<float4*>(bo.P + ri * (kC * kC) + i * kC + col0);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            float w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) w[e] = (col0 + 4 * q4 + e) < i ? v[4 * q4 + e] : 0.f;
            Pr[q4] = make_float4(w[0], w[1], w[2], w[3]);
          }
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int J = (col0 >> 4) + half;
          if (J <= I) {
            float* dst = a_blk(sm, blk(I, J));
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              float w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int jj = half * 16 + q4 * 4 + e;
                w[e] = (col0 + jj) < i ? bi * v[jj] : 0.f;
              }
              *reinterpret_cast<float4*>(dst + bidx(i & 15, q4 * 4)) = make_float4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      } else {
        const int i = row - kC;
#pragma unroll
        for (int p8 = 0; p8 < 4; ++p8) {  // row i of A_qk, 8 columns per 16-byte store
          float w8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) w8[e] = (col0 + 8 * p8 + e) <= i ? v[8 * p8 + e] : 0.f;
          st_kmajor8(sm + kP1QT, i, col0 + 8 * p8, kC, w8);
        }
      }
    }
  } else {
    // ---- exact path for chunks whose gates decay past e^-64: the score
    // matrices straight from their definition, every decay factor
    // exp(G_i - G_j) <= 1 formed per (pair, channel).  G is staged in fp32
    // one 64-channel half at a time over the dead g rows of region A.
    auto gp = [&](int i, int c) -> float* {  // c in [0, 64): channel of the staged half
      return c < 32 ? reinterpret_cast<float*>(sm + kP1A) + i * 32 + c
                    : reinterpret_cast<float*>(sm + kP1A + 16384) + i * 32 + (c - 32);
    };
    constexpr int kPairs = kC * (kC + 1) / 2;  // (i, j) with j <= i
    float akk[9], aqk[9];
#pragma unroll
    for (int t = 0; t < 9; ++t) akk[t] = aqk[t] = 0.f;
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {
      if constexpr (kMmaScan) {
        float Gq[16];
        tmem_ld16(hf == 0 ? lane_tm + kTmG0 + 16 * (warp >> 2) : lane_tm + 16 * q4, Gq);
#pragma unroll
        for (int e = 0; e < 16; ++e) *gp(mi, 16 * q4 + e) = Gq[e];
      } else if ((c8 >> 6) == hf) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          float Gt[8];
          tmem_ld8(g_tm + 8 * t, Gt);
#pragma unroll
          for (int e = 0; e < 8; ++e) *gp(tg + 16 * t, c8 - 64 * hf + e) = Gt[e];
        }
      }
      __syncthreads();
#pragma unroll 1
      for (int t = 0; t < 9; ++t) {
        const int p = tid + t * kP1Threads;
        if (p < kPairs) {
          int i = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
          while (i * (i + 1) / 2 > p) --i;
          while ((i + 1) * (i + 2) / 2 <= p) ++i;
          const int j = p - i * (i + 1) / 2;
          float sk = akk[t], sq = aqk[t];
#pragma unroll 4
          for (int c = 0; c < 64; c += 2) {
            const int ch = 64 * hf + c;
            const float2 ki = ld_bf2(sm + kP1B + kmajor_off(i, ch, kC));
            const float2 kj = ld_bf2(sm + kP1B + kmajor_off(j, ch, kC));
            const float2 qi = ld_bf2(sm + kP1A + kmajor_off(kC + i, ch, 128));
            const float d0 = __expf(*gp(i, c) - *gp(j, c)), d1 = __expf(*gp(i, c + 1) - *gp(j, c + 1));
            sk = fmaf(ki.x * kj.x, d0, fmaf(ki.y * kj.y, d1, sk));
            sq = fmaf(qi.x * kj.x, d0, fmaf(qi.y * kj.y, d1, sq));
          }
          akk[t] = sk;
          aqk[t] = sq;
        }
      }
      __syncthreads();  // this half of G is read
    }
    // pass 2 (exact): start- and end-decayed operands, factors <= 1; K+ goes
    // over the dead g rows of region A (where the factored form keeps K+_r),
    // with a unit W scale
    if constexpr (kMmaScan) {
      if (tid < kD) segr[tid] = 1.f;
#pragma unroll 1
      for (int p = 0; p < 4; ++p) {
        const int hf = p >> 1, c = 64 * hf + 16 * q4 + 8 * (p & 1);
        float Gt[8], ge[8], k8[8], q8[8], kp[8], qp[8], kb[8];
        tmem_ld8(hf == 0 ? lane_tm + kTmG0 + 16 * (warp >> 2) + 8 * (p & 1) : lane_tm + 16 * q4 + 8 * (p & 1), Gt);
        const uint32_t oK = kmajor_off(mi, c, kC);
        ld8(sm + kP1B + oK, k8);
        ld8(sm + kP1A + kmajor_off(kC + mi, c, 128), q8);
        {
          const float4 a0 = *reinterpret_cast<const float4*>(sgend + c), a1 = *reinterpret_cast<const float4*>(sgend + c + 4);
          ge[0] = a0.x, ge[1] = a0.y, ge[2] = a0.z, ge[3] = a0.w, ge[4] = a1.x, ge[5] = a1.y, ge[6] = a1.z, ge[7] = a1.w;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float e0 = __expf(Gt[e]);
          kp[e] = k8[e] * e0;
          qp[e] = scale * q8[e] * e0;
          kb[e] = k8[e] * __expf(ge[e] - Gt[e]);
        }
        st8(sm + kP1A + kmajor_off(mi, c, 128), kp);
        st8(rec + oRecQ + oK, qp);
        st8(rec + oRecKbar + oK, kb);
      }
    } else {
      if (tg == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) segr[c8 + e] = 1.f;
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int i = tg + 16 * t;
        const uint32_t oK = kmajor_off(i, c8, kC);
        const uint32_t oQ = kmajor_off(kC + i, c8, 128);
        float k8[8], q8[8], kp[8], qp[8], kb[8], Gt[8];
        tmem_ld8(g_tm + 8 * t, Gt);
        ld8(sm + kP1B + oK, k8);
        ld8(sm + kP1A + oQ, q8);
        if (l2n) {
          const float rk = rsqrtf(snk[i] + kL2Eps), rq = rsqrtf(snq[i] + kL2Eps);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            k8[e] *= rk;
            q8[e] *= rq;
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float e0 = __expf(Gt[e]);
          kp[e] = k8[e] * e0;
          qp[e] = scale * q8[e] * e0;
          kb[e] = k8[e] * __expf(gend[e] - Gt[e]);
        }
        st8(sm + kP1A + kmajor_off(i, c8, 128), kp);
        st8(rec + oRecQ + oK, qp);
        st8(rec + oRecKbar + oK, kb);
      }
    }
    __syncthreads();  // k and q are read: region B takes the A_kk blocks, [24K,32K) of region A the A_qk staging
#pragma unroll 1
    for (int t = 0; t < 9; ++t) {
      const int p = tid + t * kP1Threads;
      if (p < kPairs) {
        int i = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
        while (i * (i + 1) / 2 > p) --i;
        while ((i + 1) * (i + 2) / 2 <= p) ++i;
        const int j = p - i * (i + 1) / 2;
        float fk = 1.f, fq = 1.f;  // unit-length factors of k_i k_j and q_i k_j
        if (l2n) {
          const float rkj = rsqrtf(snk[j] + kL2Eps);
          fk = rsqrtf(snk[i] + kL2Eps) * rkj;
          fq = rsqrtf(snq[i] + kL2Eps) * rkj;
        }
        a_blk(sm, blk(i >> 4, j >> 4))[bidx(i & 15, j & 15)] = j < i ? sbeta[i] * (akk[t] * fk) : 0.f;
        if (kBwd) bo.P[ri * (kC * kC) + i * kC + j] = j < i ? akk[t] * fk : 0.f;
        stbf(sm + kP1QT, kmajor_off(i, j, kC), scale * (aqk[t] * fq));
      }
    }
    for (int e = tid; e < kC * kC; e += kP1Threads) {
      const int i = e / kC, j = e % kC;
      if (j > i) {
        stbf(sm + kP1QT, kmajor_off(i, j, kC), 0.f);
        if (kBwd) bo.P[ri * (kC * kC) + e] = 0.f;
      }
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    bulk_store(rec + oRecAqk, sm + kP1QT, 8192);
    bulk_commit();
    // Q+_r is dead: bring v while the triangle is inverted, its first
    // channel half now, the second once the A_qk store has read its bytes
    mbar_expect_tx(&bar_v, 16384);
    tma_load_4d(sm + kP1V, &tm_v, &bar_v, 0, h, t0, b);
  }

  // ---- T = (I + A_kk)^-1 by 16 x 16 blocks, fp32
  if (tid < 64) {  // diagonal blocks by forward substitution, one column per thread
    const int I = tid >> 4, jj = tid & 15;
    const float* A = a_blk(sm, blk(I, I));
    float t[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < r; ++m) acc = fmaf(A[bidx(r, m)], t[m], acc);
      t[r] = r < jj ? 0.f : (r == jj ? 1.f : -acc);
    }
    float* Tb = t_blk(sm, blk(I, I));
#pragma unroll
    for (int r = 0; r < 16; ++r) Tb[bidx(r, jj)] = t[r];
  }
  __syncthreads();
  if (tid == 0) {
    bulk_wait_read();
    tma_load_4d(sm + kP1V + 16384, &tm_v, &bar_v, 64, h, t0, b);
  }
  // off-diagonal blocks, one sub-diagonal at a time, one warp per block:
  //   X = sum_{K=J}^{I-1} A_IK T_KJ,   T_IJ = -T_II X
  // as 16x16x16 products on the warp-level tensor cores (tf32 in, fp32
  // accumulate; the result is rounded to bf16 for the W/U MMAs afterwards).
#pragma unroll 1
  for (int d = 1; d < 4; ++d) {
    if (warp < 4 - d) {
      const int J = warp, I = J + d;
      float* Tij = t_blk(sm, blk(I, J));
      float x[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      for (int K = J; K < I; ++K) block_mma_tf32(x, a_blk(sm, blk(I, K)), t_blk(sm, blk(K, J)), lane);
      store_block_frag(Tij, x, lane, 1.f);  // X parked in the slot of T_IJ
      __syncwarp();
      float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      block_mma_tf32(y, t_blk(sm, blk(I, I)), Tij, lane);
      __syncwarp();
      store_block_frag(Tij, y, lane, -1.f);
    }
    __syncthreads();
  }
  // (T diag(beta))^T as the K-major B operand of the W/U MMAs: row n = i, column k = j
  // (over the A_kk blocks, read by now).
  {
    const int i = tid >> 2, j0 = (tid & 3) * 16, I = i >> 4, J = j0 >> 4;
    float vals[16];
    if (J <= I) {
      const float* Tb = t_blk(sm, blk(I, J));
      if (kBwd) {  // T itself, row i, columns j0 .. j0 + 15, bf16
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) vals[jj] = (j0 + jj) <= i ? Tb[bidx(i & 15, jj)] : 0.f;
        uint4* Tr = reinterpret_cast<uint4*>(bo.T + ri * (kC * kC) + i * kC + j0);
        Tr[0] = make_uint4(pack2(vals[0], vals[1]), pack2(vals[2], vals[3]), pack2(vals[4], vals[5]),
                           pack2(vals[6], vals[7]));
        Tr[1] = make_uint4(pack2(vals[8], vals[9]), pack2(vals[10], vals[11]), pack2(vals[12], vals[13]),
                           pack2(vals[14], vals[15]));
      }
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) vals[jj] = (j0 + jj) <= i ? Tb[bidx(i & 15, jj)] * sbeta[j0 + jj] : 0.f;
    } else {
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) vals[jj] = 0.f;
      if (kBwd) {
        uint4* Tr = reinterpret_cast<uint4*>(bo.T + ri * (kC * kC) + i * kC + j0);
        Tr[0] = Tr[1] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    st_kmajor8(sm + kP1B2, i, j0, kC, vals);
    st_kmajor8(sm + kP1B2, i, j0 + 8, kC, vals + 8);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- W^T / segr = K+_r^T (T diag beta)^T, U^T = V^T (T diag beta)^T  (M=128, N=64, K=64).
  // K+_r = K+ / exp(G_r) per channel (rows 0-63 of region A, channel halves
  // 16 KiB apart; K+ itself on the exact path, segr = 1), so the extraction
  // scales row c of the first product by segr[c]; v's halves are 16 KiB apart too.
  if (tid == 0) {
    wait_or_flag(&bar_v, 0, hdr, 3);
    tc_fence_after();
    const uint32_t idesc = idesc_bf16_f32(128, 64, 1, 0);
    const uint32_t kb = smem_u32(sm + kP1A), vb = smem_u32(sm + kP1V), b2 = smem_u32(sm + kP1B2);
#pragma unroll
    for (int k = 0; k < kC / 16; ++k) {
      const uint64_t bd = desc_sw128(b2 + k * 32, 16, 1024);
      mma_bf16(tm, desc_sw128(kb + 2 * k * 1024, 16384, 1024), bd, idesc, k > 0);
      mma_bf16(tm + 64, desc_sw128(vb + 2 * k * 1024, 16384, 1024), bd, idesc, k > 0);
    }
    mma_commit(&bar_mma);
  }
  wait_or_flag(&bar_mma, slow ? 0 : 1, hdr, 4);
  tc_fence_after();

  // ---- -W^T (channel rows over the first 16 KiB of region A, dead once the
  // W/U products are done: row c, 64 tokens) and U^T (region B, 128-row K-major)
  {
    const int c = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const float wsc = warp < 4 ? (kBwd ? segr[c] : -segr[c]) : 0.f;
    float v[32];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      if (warp < 4) {
        tmem_ld32(tm + lane_off + half * 32, v);
        if (kBwd) {  // W as token rows: element (token, channel c) of the 64 x 128 tile
#pragma unroll
          for (int e = 0; e < 32; ++e) stbf(sm + kP1A, kmajor_off(half * 32 + e, c, kC), wsc * v[e]);
        } else {
#pragma unroll
          for (int p8 = 0; p8 < 4; ++p8) {
            float w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w8[e] = wsc * v[8 * p8 + e];
            st_kmajor8(sm + kP1A, c, half * 32 + 8 * p8, 128, w8);
          }
        }
      } else {
        tmem_ld32(tm + lane_off + 64 + half * 32, v);
        if (kBwd) {  // U[token][c], fp32: a warp writes 32 consecutive channels of a token row
          float* Ur = bo.U + ri * (kC * kD) + (size_t)(half * 32) * kD + c;
#pragma unroll
          for (int e = 0; e < 32; ++e) Ur[e * kD] = v[e];
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) st_kmajor8(sm + kP1B, c, half * 32 + 8 * e, 128, v + 8 * e);
        }
      }
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    if (kBwd) {
      bulk_store(rec + kTcRecW, sm + kP1A, 16384);
    } else {
      bulk_store(rec + kRecW, sm + kP1A, 16384);
      bulk_store(rec + kRecU, sm + kP1B, 16384);
    }
    bulk_commit();
    bulk_wait_read();
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 128);
}

// =============================================================== kernel 2
// Warp roles (288 threads):
//   warps 0-3  "state":  the sequential chain.  Thread j owns TMEM lane j =
//              value channel j (row j of S^T); they convert S0^T and V'^T to
//              bf16 MMA operands and decay S^T in place.
//   warps 4-7  "output": read O^T of each chunk from TMEM, stage it in shared
//              memory and store it with two TMA tile stores (scattered 2-byte
//              global stores from these warps were found to slow the tensor
//              pipe down by half).
//   warp  8    "mma":    one thread issues every tcgen05.mma (an issue costs
//              tens of cycles, so the issuer gets a warp of its own).
//   Thread 128 also streams the per-chunk records into two stages; it issues
//   each copy only after releasing O^T, since a bulk-copy issue holds up its
//   warp and the MMA warp waits for that release.
// Tensor memory (fp32 unless noted):
//   [P | O^T | S^T] at [0,64) [64,128) [128,256)
//   S0^T as bf16 A operand [256,320), V'^T as bf16 A operand [320,352)
// Four MMA groups per chunk, all A operands read from tensor memory:
//   P    = S0^T (-W)^T     (N = 64,  K = 128: 8 instructions, committed alone; B = -W^T, MN-major)
//   O^T  = S0^T Q+^T       (N = 64,  K = 128: 8 instructions, while V' is formed; B = Q+, K-major)
//   O^T += V'^T A_qk^T     (N = 64,  K = 64:  4 instructions; B = A_qk, K-major)
//   S^T += V'^T Kbar       (N = 128, K = 64:  4 instructions; B = Kbar, MN-major)
// with P = -(W S0)^T and V'^T = U^T + P formed on the CUDA cores.  Only P
// and the S^T update are on the chain's critical path; the O^T groups wait
// for the output warps to release the previous chunk's O^T off that path.
constexpr int kSPThreads = 288;
constexpr uint32_t kTmP = 0, kTmO = 64, kTmS = 128, kTmAS = 256, kTmAV = 320;

// The passes without outputs (the scan's offset and transition passes) run
// a lighter instance of the same kernel, two CTAs per SM: 192 threads (state
// warps 0-3, warp 4 streams the records, warp 5 issues the MMAs), 256 columns
// of tensor memory ([P | S^T | S0^T bf16], V'^T in bf16 written over the P
// columns it was formed from), compact stages holding only -W^T, Kbar, U
// and gamma, and the start state
// read straight from global memory.
constexpr int kSPThreadsNoOut = 192;
constexpr uint32_t kTmSNo = 64, kTmASNo = 192;  // P at 0, V'^T bf16 over P's first 32 columns
constexpr uint32_t kCW = 0, kCKbar = 16384, kCU = 32768, kCGamma = 49152;  // compact stage offsets
constexpr uint32_t kStageNoOut = 50176;      // 49 KiB
constexpr uint32_t kP2BytesNoOut = 2 * kStageNoOut;
static_assert(kCGamma + 512 <= kStageNoOut, "compact stage");

// Brings the record of one chunk into a stage.  A pass that writes outputs
// needs all of it; a pass without outputs reads only -W^T, Kbar, U and
// gamma; the transition pass (U = 0) not even U.
constexpr uint32_t kRecNoOutBytes = (kRecQ - kRecW) + (kRecBytes - kRecKbar);
constexpr uint32_t kRecTransBytes = (kRecQ - kRecW) + (kRecU - kRecKbar) + (kRecBytes - kRecGamma);
__device__ __forceinline__ void load_record(uint8_t* stage, const uint8_t* rec, uint64_t* bar, bool out,
                                            bool zero_u) {
  if (out) {
    mbar_expect_tx(bar, kRecBytes);
    bulk_load(stage, rec, kRecBytes, bar);
    return;
  }
  mbar_expect_tx(bar, zero_u ? kRecTransBytes : kRecNoOutBytes);
  bulk_load(stage + kRecW, rec + kRecW, kRecQ - kRecW, bar);
  if (zero_u) {
    bulk_load(stage + kRecKbar, rec + kRecKbar, kRecU - kRecKbar, bar);
    bulk_load(stage + kRecGamma, rec + kRecGamma, kRecBytes - kRecGamma, bar);
  } else {
    bulk_load(stage + kRecKbar, rec + kRecKbar, kRecBytes - kRecKbar, bar);
  }
}

// The same parts into a compact stage: -W^T to [0, 16K), then Kbar, U and
// gamma, contiguous in the record, to [16K, 48.5K) (U skipped for the
// transition pass).
__device__ __forceinline__ void load_record_compact(uint8_t* stage, const uint8_t* rec, uint64_t* bar, bool zero_u) {
  mbar_expect_tx(bar, zero_u ? kRecTransBytes : kRecNoOutBytes);
  bulk_load(stage + kCW, rec + kRecW, kRecQ - kRecW, bar);
  if (zero_u) {
    bulk_load(stage + kCKbar, rec + kRecKbar, kRecU - kRecKbar, bar);
    bulk_load(stage + kCGamma, rec + kRecGamma, kRecBytes - kRecGamma, bar);
  } else {
    bulk_load(stage + kCKbar, rec + kRecKbar, kRecBytes - kRecKbar, bar);
  }
}
static_assert(kCU - kCKbar == kRecU - kRecKbar && kCGamma - kCKbar == kRecGamma - kRecKbar, "compact = record order");

// What one state-pass CTA does.  Phase 0: a whole chain.  With the
// chunk-parallel scan (few chains, long sequences) a chain is cut into G
// groups of L chunks; phase 1 runs, per group, a zero-start pass whose final
// state is R_g (group 0 starts from the true initial state instead) and an
// identity-start pass with U = 0 whose final state is the group's transition
// M_g (S_end = M_g S_start + R_g, the map is affine in S_start); phase 3 runs
// every group again from its true start state S_g (computed in between by
// kda_scan_combine_kernel) and writes the outputs.
// The caller's states are [B*H][dk][dv] (dk, dv in {64, 128}); inside the
// kernels every state is 128 x 128, the channels past dk (dv) being zero.
// The scan buffers use that internal layout: R_g in rbuf, the transitions
// in mbuf, and in sbuf the start state of group 0 (slot 0, copied there by
// phase 1, so that phase 3 never reads the caller's initial state, which
// the caller's final state may overwrite) and of groups 2..G-1.
struct StatePassArgs {
  const uint8_t* records;
  WorkspaceHeader* hdr;
  const float* s0;  // [B*H][dk][dv] or null (zero)
  float* sT;        // [B*H][dk][dv] or null
  float* rbuf;      // [B*H][G][128][128] scan buffers
  float* mbuf;      // transition matrices: [B*H][G] slots of 64 KiB, each the 32 KiB bf16 K-major image of M_g
  float* sbuf;
  int T, H, NC, G, L, phase, dk, dv;
  // phase 3 launches may cover groups [g_first, g_first + g_count) only (0: all);
  // s0_direct: group 0 reads the caller's initial state itself; dep_wait = 0:
  // no wait for the previous grid (its inputs were complete before that grid
  // could be scheduled); trigger: let the next grid be scheduled early
  int g_first, g_count, s0_direct, dep_wait, trigger;
};

template <bool kOut>
__global__ void __launch_bounds__(kOut ? kSPThreads : kSPThreadsNoOut, kOut ? 1 : 2)
    kda_state_pass_kernel(const __grid_constant__ CUtensorMap tm_o, const StatePassArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ uint64_t bar_full[2], bar_o, bar_p, bar_s, bar_as, bar_av, bar_init;
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, warp = tid >> 5;
  WorkspaceHeader* hdr = args.hdr;
  const int H = args.H, NC = args.NC, G = args.G, L = args.L;
  constexpr size_t kSt = (size_t)kD * kD;
  // ---- role of this CTA
  const int dk = args.dk, dv = args.dv;
  const size_t kUserSt = (size_t)dk * dv;
  int bh, cb, ce;
  const float* init = nullptr;  // null: zero start
  bool ident = false, zero_u = false;
  // Phases 0 and 3 write outputs (full instance).  Phase 1 writes none: the
  // light instance for long chains, the full one otherwise.
  const bool out = kOut && args.phase != 1;
  constexpr uint32_t kStg = kOut ? kStage : kStageNoOut;
  constexpr int kMmaWarp = kOut ? 8 : 5;
  constexpr uint32_t tP = kTmP, tS = kOut ? kTmS : kTmSNo, tAS = kOut ? kTmAS : kTmASNo, tAV = kOut ? kTmAV : kTmP;
  bool init_user = false, fin_user = false;  // caller's [dk][dv] layout (else the internal 128 x 128)
  float* fin = nullptr;
  float* init_copy = nullptr;  // phase 1, group 0: the start state is also kept in sbuf slot 0
  if (args.phase == 0) {
    bh = blockIdx.x;
    cb = 0;
    ce = NC;
    init = args.s0 ? args.s0 + bh * kUserSt : nullptr;
    fin = args.sT ? args.sT + bh * kUserSt : nullptr;
    init_user = fin_user = true;
  } else if (args.phase == 1) {
    const int per = 2 * G - 3;
    bh = blockIdx.x / per;
    const int r = blockIdx.x % per;
    int g;
    if (r < G - 1) {
      g = r;
      init = (g == 0 && args.s0) ? args.s0 + bh * kUserSt : nullptr;
      init_user = true;
      if (g == 0 && args.s0) init_copy = args.sbuf + (size_t)bh * G * kSt;
      fin = args.rbuf + ((size_t)bh * G + g) * kSt;
    } else {
      g = r - (G - 1) + 1;
      ident = true;
      zero_u = true;
      fin = args.mbuf + ((size_t)bh * G + g) * kSt;
    }
    cb = g * L;
    ce = min(NC, cb + L);
  } else {
    const int gn = args.g_count > 0 ? args.g_count : G;
    bh = blockIdx.x / gn;
    const int g = args.g_first + blockIdx.x % gn;
    cb = g * L;
    ce = min(NC, cb + L);
    // group 0 starts from the initial state (the caller's, or its copy in sbuf
    // slot 0), group 1 from R_0; later ones from the combination kernel's output
    if (g == 0 && args.s0_direct) {
      init = args.s0 ? args.s0 + bh * kUserSt : nullptr;
      init_user = true;
    } else {
      init = g == 0 ? (args.s0 ? args.sbuf + (size_t)bh * G * kSt : nullptr)
                    : g == 1 ? args.rbuf + (size_t)bh * G * kSt : args.sbuf + ((size_t)bh * G + g) * kSt;
    }
    fin = (g == G - 1 && args.sT) ? args.sT + bh * kUserSt : nullptr;
    fin_user = true;
  }
  const int NCL = ce - cb;  // chunks this CTA walks
  const int h = bh % H, b = bh / H;
  const uint8_t* recs = args.records + ((size_t)bh * NC + cb) * kRecBytes;

  // Launched right behind the kernel that wrote its inputs: nothing global
  // (and no tensor memory, which that kernel's CTAs may still be allocating)
  // is touched before it has finished.
  if (tid == 0) prefetch_tensormap(&tm_o);
  if (args.dep_wait) grid_dep_wait();
  if (tid == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(&bar_o, 1);
    mbar_init(&bar_p, 1);
    mbar_init(&bar_s, 1);
    mbar_init(&bar_as, out ? 256 : 128);  // with outputs the output warps release O^T through it too
    mbar_init(&bar_av, 128);
    mbar_init(&bar_init, 1);
    fence_mbar_init();
    if (kOut && init) {  // the start state, row-major fp32, into stage 1 (its record follows once it is read)
      const uint32_t bytes = (uint32_t)((init_user ? kUserSt : kSt) * sizeof(float));  // 16, 32 or 64 KiB
      mbar_expect_tx(&bar_init, bytes);
      for (uint32_t p = 0; p < bytes / 16384; ++p)
        bulk_load(sm + kStage + p * 16384, init + p * 4096, 16384, &bar_init);
    }
  }
  if (warp == 0) tmem_alloc(&tmem_base, kOut ? 512 : 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_base;
  if (args.phase == 1 || args.trigger) grid_dep_launch();  // the next kernel may be scheduled

  if (warp == kMmaWarp) {
    // ------------------------------------------------------------ mma
    if ((tid & 31) == 0) {
      // P = S0^T (-W)^T (N=64) first, committed alone so that V' can be formed
      // at once; with outputs, O^T = S0^T Q+^T (N=64) is issued next, while
      // the state warps form V'; then O^T += V'^T A_qk^T (N=64) and
      // S^T += V'^T Kbar (N=128) close the chunk (without outputs only the last).
      const uint32_t id_w = idesc_bf16_f32(128, 64, 0, 1);    // B = -W^T, MN-major (N = tokens)
      const uint32_t id_k = idesc_bf16_f32(128, 64, 0, 0);    // B = Q+ or A_qk rows, K-major
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 1);   // B = Kbar, MN-major (N = channels)
      // first descriptors of each stage; later steps add address offsets (in 16-byte units)
      const uint32_t oW = kOut ? kRecW : kCW, oK = kOut ? kRecKbar : kCKbar;
      auto desc_at = [&](int s, uint32_t off, uint32_t lbo) { return desc_sw128(smem_u32(sm + s * kStg + off), lbo, 1024); };
      const uint64_t dw0 = desc_at(0, oW, 8192), dw1 = desc_at(1, oW, 8192);
      const uint64_t dk0 = desc_at(0, oK, 8192), dk1 = desc_at(1, oK, 8192);
      const uint64_t dq0 = desc_at(0, kRecQ, 16), dq1 = desc_at(1, kRecQ, 16);      // with outputs only
      const uint64_t da0 = desc_at(0, kRecAqk, 16), da1 = desc_at(1, kRecAqk, 16);  // with outputs only
      for (int n = 0; n < NCL; ++n) {
        const int s = n & 1;
        const uint64_t dws = s ? dw1 : dw0, dks = s ? dk1 : dk0, dqs = s ? dq1 : dq0, das = s ? da1 : da0;
        wait_or_flag(&bar_as, n & 1, hdr, 30);
        wait_or_flag(&bar_full[s], (n >> 1) & 1, hdr, 31);
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kD / 16; ++k)  // MN-major B: 16 channel rows (2 KiB) per step
          mma_bf16_ts(tm + tP, tm + tAS + k * 8, dws + (uint64_t)((k * 2048) >> 4), id_w, k > 0);
        mma_commit(&bar_p);
        if (out) {  // bar_as also covered the read of O^T of chunk n-1
#pragma unroll
          for (int k = 0; k < kD / 16; ++k)  // K-major B (64 token rows): +32 B per step, +8 KiB per 64-channel block
            mma_bf16_ts(tm + kTmO, tm + tAS + k * 8, dqs + (uint64_t)(((k / 4) * 8192 + (k % 4) * 32) >> 4), id_k,
                        k > 0);
        }
        wait_or_flag(&bar_av, n & 1, hdr, 33);
        tc_fence_after();
        if (out) {
#pragma unroll
          for (int k = 0; k < kC / 16; ++k)  // K-major B (rows i): 16 tokens j = 32 B per step
            mma_bf16_ts(tm + kTmO, tm + tAV + k * 8, das + (uint64_t)((k * 32) >> 4), id_k, 1);
        }
#pragma unroll
        for (int k = 0; k < kC / 16; ++k)  // MN-major B: +2 KiB per 16 K-rows
          mma_bf16_ts(tm + tS, tm + tAV + k * 8, dks + (uint64_t)((2 * k * 1024) >> 4), id_s, 1);
        mma_commit(&bar_s);
        mma_commit(&bar_o);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ output + loads
    const int j = tid - 128;
    const uint32_t lane_off = (uint32_t)((warp - 4) * 32) << 16;
    if (tid == 128) {
      for (int n = 0; n < 2 && n < NCL; ++n) {
        if (!kOut)
          load_record_compact(sm + n * kStg, recs + (size_t)n * kRecBytes, &bar_full[n], zero_u);
        else if (n == 0 || !init)
          load_record(sm + n * kStage, recs + (size_t)n * kRecBytes, &bar_full[n], out, zero_u);
      }
    }
    // With outputs, each chunk's bar_as phase also waits for these 128
    // threads: the first has nothing to release, later ones the O^T of the
    // chunk before (whose O^T group overwrites it).
    if (out) mbar_arrive(&bar_as);
    for (int n = 0; n < NCL; ++n) {
      const int s = n & 1;
      wait_or_flag(&bar_o, n & 1, hdr, 21);
      tc_fence_after();
      if (!out) {
        if (tid == 128 && n + 2 < NCL) {
          if (kOut)
            load_record(sm + s * kStage, recs + (size_t)(n + 2) * kRecBytes, &bar_full[s], false, zero_u);
          else
            load_record_compact(sm + s * kStg, recs + (size_t)(n + 2) * kRecBytes, &bar_full[s], zero_u);
        }
        continue;
      }
      uint32_t r[64];
      tmem_ld32_raw(tm + kTmO + lane_off, r);
      tmem_ld32_raw(tm + kTmO + lane_off + 32, r + 32);
      tmem_wait_ld();
      reg_pin<64>(r);
      tc_fence_before();
      if (n + 1 < NCL) mbar_arrive(&bar_as);
      if (tid == 128 && n + 2 < NCL) {  // every reader of stage s is done with chunk n
        mbar_expect_tx(&bar_full[s], kRecBytes);
        bulk_load(sm + s * kStage, recs + (size_t)(n + 2) * kRecBytes, kRecBytes, &bar_full[s]);
      }
      // staging tile n%2 must no longer be read by the TMA store of chunk n-2
      if (tid == 128) bulk_wait_read_n<1>();
      named_bar_sync(2, 128);
      uint8_t* stg = sm + kP2Out + (n & 1) * 16384 + (j >> 6) * 8192 + (j & 63) * 2;
#pragma unroll
      for (int i = 0; i < kC; ++i)
        *reinterpret_cast<bf16*>(stg + i * 128) = __float2bfloat16_rn(__uint_as_float(r[i]));
      fence_async_smem();
      named_bar_sync(2, 128);
      if (tid == 128) {
        const uint8_t* src = sm + kP2Out + (n & 1) * 16384;
        tma_store_4d(&tm_o, src, 0, h, (cb + n) * kC, b);
        if (dv > 64) tma_store_4d(&tm_o, src + 8192, 64, h, (cb + n) * kC, b);
        bulk_commit();
      }
    }
    if (tid == 128) bulk_wait_read_n<0>();
  } else {
    // ------------------------------------------------------------ state
    const int j = tid;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    {
      // column j of the start state (row j of S^T) into lane j: from stage 1
      // (with outputs) or straight from global memory (without)
      const float* s0s = kOut ? reinterpret_cast<const float*>(sm + kStage) : init;
      if (kOut && init) wait_or_flag(&bar_init, 0, hdr, 20);
      float v[32];
#pragma unroll
      for (int q = 0; q < kD / 32; ++q) {
#pragma unroll
        for (int ii = 0; ii < 32; ++ii) {
          const int c = q * 32 + ii;
          if (!init)
            v[ii] = ident && c == j ? 1.f : 0.f;
          else if (init_user)
            v[ii] = (c < dk && j < dv) ? s0s[c * dv + j] : 0.f;
          else
            v[ii] = s0s[c * kD + j];
          if (init_copy) init_copy[(size_t)c * kD + j] = v[ii];
        }
        tmem_st32(tm + tS + lane_off + q * 32, v);
      }
      tmem_wait_st();
      if (kOut && init) {  // stage 1 is free again: bring the record of chunk 1
        named_bar_sync(1, 128);
        if (tid == 0 && NCL > 1) load_record(sm + kStage, recs + kRecBytes, &bar_full[1], out, zero_u);
      }
    }
    constexpr uint32_t oU = kOut ? kRecU : kCU, oGam = kOut ? kRecGamma : kCGamma;
    for (int n = 0; n < NCL; ++n) {
      const int s = n & 1;
      const uint8_t* stage = sm + s * kStg;
      if (n > 0) wait_or_flag(&bar_s, (n - 1) & 1, hdr, 22);
      tc_fence_after();

      // (1) S0^T -> bf16 A operand in tensor memory, 64 columns at a time
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t sr[64];
        tmem_ld32_raw(tm + tS + lane_off + half * 64, sr);
        tmem_ld32_raw(tm + tS + lane_off + half * 64 + 32, sr + 32);
        tmem_wait_ld();
        reg_pin<64>(sr);
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) pk[e] = pack2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]));
        tmem_st32u(tm + tAS + lane_off + half * 32, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_as);

      // (2) S^T <- S^T Diag(gamma) while the MMAs run
      wait_or_flag(&bar_full[s], (n >> 1) & 1, hdr, 25);
      {
        const float4* gam = reinterpret_cast<const float4*>(stage + oGam);
#pragma unroll
        for (int cb = 0; cb < kD / 32; ++cb) {
          uint32_t sr[32];
          tmem_ld32_raw(tm + tS + lane_off + cb * 32, sr);
          tmem_wait_ld();
          reg_pin<32>(sr);
          float v[32];
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 gg = gam[cb * 8 + q4];
            v[q4 * 4 + 0] = __uint_as_float(sr[q4 * 4 + 0]) * gg.x;
            v[q4 * 4 + 1] = __uint_as_float(sr[q4 * 4 + 1]) * gg.y;
            v[q4 * 4 + 2] = __uint_as_float(sr[q4 * 4 + 2]) * gg.z;
            v[q4 * 4 + 3] = __uint_as_float(sr[q4 * 4 + 3]) * gg.w;
          }
          tmem_st32(tm + tS + lane_off + cb * 32, v);
        }
      }

      // (3) V'^T = U^T + P -> bf16 A operand in tensor memory, 32 columns at a time
      uint4 urow[4];
#pragma unroll
      for (int k8 = 0; k8 < 4; ++k8)
        urow[k8] = *reinterpret_cast<const uint4*>(stage + oU + kmajor_off(j, k8 * 8, kD));
      wait_or_flag(&bar_p, n & 1, hdr, 26);
      tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pr[32];
        tmem_ld32_raw(tm + tP + lane_off + half * 32, pr);
        tmem_wait_ld();
        reg_pin<32>(pr);
        uint32_t pk[16];
#pragma unroll
        for (int k8 = 0; k8 < 4; ++k8) {
          const uint32_t uw[4] = {urow[k8].x, urow[k8].y, urow[k8].z, urow[k8].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float2 u2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&uw[e]));
            if (zero_u) u2 = make_float2(0.f, 0.f);
            pk[k8 * 4 + e] = pack2(u2.x + __uint_as_float(pr[k8 * 8 + 2 * e]),
                                   u2.y + __uint_as_float(pr[k8 * 8 + 2 * e + 1]));
          }
        }
        if (half == 0) {
#pragma unroll
          for (int k8 = 0; k8 < 4; ++k8)
            urow[k8] = *reinterpret_cast<const uint4*>(stage + oU + kmajor_off(j, 32 + k8 * 8, kD));
        }
        // without outputs V'^T goes over the P columns this thread has just read
        tmem_st16u(tm + tAV + lane_off + half * 16, pk);
      }
      tmem_wait_st();  // also covers the decayed S^T
      tc_fence_before();
      mbar_arrive(&bar_av);
    }
    wait_or_flag(&bar_s, (NCL - 1) & 1, hdr, 27);
    tc_fence_after();
    if (fin) {
#pragma unroll
      for (int q = 0; q < kD / 32; ++q) {
        float v[32];
        tmem_ld32(tm + tS + lane_off + q * 32, v);
        if (ident) {
          // A transition matrix is stored as the bf16 K-major 128-row image of
          // M (row r, column j at kmajor_off(r, j)), the B operand of the
          // combination kernel; this thread holds column j.
          uint8_t* img = reinterpret_cast<uint8_t*>(fin);
#pragma unroll
          for (int ii = 0; ii < 32; ++ii) stbf(img, kmajor_off(q * 32 + ii, j, kD), v[ii]);
        } else if (fin_user) {
          if (j < dv) {
#pragma unroll
            for (int ii = 0; ii < 32; ++ii)
              if (q * 32 + ii < dk) fin[(size_t)(q * 32 + ii) * dv + j] = v[ii];
          }
        } else {
#pragma unroll
          for (int ii = 0; ii < 32; ++ii) fin[(size_t)(q * 32 + ii) * kD + j] = v[ii];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem_base, kOut ? 512 : 256);
}

// ======================================================== scan combine
// S_{g+1} = M_g S_g + R_g for g = 1 .. G-2 (S_1 = R_0; the output pass reads
// S_0 and S_1 from the initial state and from R_0 itself), one CTA per chain,
// on the tensor cores in the state pass's transposed form
//   S_{g+1}^T = S_g^T M_g^T + R_g^T:
// thread n owns TMEM lane n (value channel n); the accumulator starts as
// R_g^T, A is S_g^T in bf16 (tensor memory), B the bf16 K-major image of M_g
// written by the transition pass (rows = rows of M_g).  S and M are rounded
// to bf16 with fp32 accumulation, as in one chunk step of the state pass.
// M_g images and R_g (fp32, row-major) stream through two-stage rings.
constexpr int kCbThreads = 128;
constexpr uint32_t kCbImg = 32768;             // bytes of one M_g image
constexpr uint32_t kCbR = 65536;               // bytes of one R_g
constexpr uint32_t kCbTmS = 0, kCbTmA = 128;   // TMEM: S^T fp32 [0,128), S^T bf16 [128,192)
constexpr size_t kCbSmem = 2 * kCbImg + 2 * kCbR + 1024;

__global__ void __launch_bounds__(kCbThreads) kda_scan_combine_kernel(float* sbuf, const float* rbuf,
                                                                      const float* mbuf, int G, WorkspaceHeader* hdr) {
  extern __shared__ uint8_t cb_raw[];
  uint8_t* sm = align1024(cb_raw);  // [2 M images][2 R stages]
  __shared__ uint64_t bar_m[2], bar_r[2], bar_mma;
  __shared__ uint32_t tmem_base;
  constexpr size_t kSt = (size_t)kD * kD;
  const int tid = threadIdx.x, warp = tid >> 5, n = tid;
  const int bh = blockIdx.x;
  const float* rb = rbuf + (size_t)bh * G * kSt;
  float* sb = sbuf + (size_t)bh * G * kSt;
  const uint8_t* mb = reinterpret_cast<const uint8_t*>(mbuf + (size_t)bh * G * kSt);  // slot g at g * kSt floats
  const int nsteps = G - 2;
  auto m_img = [&](int st) { return sm + st * kCbImg; };
  auto r_tile = [&](int st) { return reinterpret_cast<const float*>(sm + 2 * kCbImg + st * kCbR); };
  auto load_m = [&](int st, int g) {
    mbar_expect_tx(&bar_m[st], kCbImg);
    bulk_load(sm + st * kCbImg, mb + (size_t)g * kSt * sizeof(float), kCbImg, &bar_m[st]);
  };
  auto load_r = [&](int st, int g) {
    mbar_expect_tx(&bar_r[st], kCbR);
#pragma unroll
    for (int p = 0; p < 4; ++p)
      bulk_load(sm + 2 * kCbImg + st * kCbR + p * (kCbR / 4), rb + (size_t)g * kSt + p * (kSt / 4), kCbR / 4,
                &bar_r[st]);
  };
  grid_dep_wait();  // the transition and offset passes have finished
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_m[i], 1);
      mbar_init(&bar_r[i], 1);
    }
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
    load_r(0, 0);                        // R_0 = S_1, the first A operand
    load_r(1, 1);
    for (int st = 0; st < 2 && st < nsteps; ++st) load_m(st, 1 + st);
  }
  if (warp == 0) tmem_alloc(&tmem_base, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_launch();  // the output pass may be scheduled (it waits for this grid)
  const uint32_t tm = tmem_base, lane_off = (uint32_t)(warp * 32) << 16;

  // A <- S_1^T = R_0^T in bf16 (row k of R_0 at k * 128 floats; thread n reads column n)
  wait_or_flag(&bar_r[0], 0, hdr, 40);
#pragma unroll
  for (int q = 0; q < kD / 32; ++q) {
    const float* r = r_tile(0) + (size_t)q * 32 * kD + n;
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) pk[e] = pack2(r[(2 * e) * kD], r[(2 * e + 1) * kD]);
    tmem_st16u(tm + kCbTmA + lane_off + q * 16, pk);
  }
  const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
  for (int step = 0; step < nsteps; ++step) {
    const int g = step + 1, s = step & 1, rs = g & 1;  // R_g sits in stage g % 2
    // accumulator <- R_g^T
    wait_or_flag(&bar_r[rs], (g >> 1) & 1, hdr, 43);
#pragma unroll
    for (int q = 0; q < kD / 32; ++q) {
      const float* r = r_tile(rs) + (size_t)q * 32 * kD + n;
      float v[32];
#pragma unroll
      for (int ii = 0; ii < 32; ++ii) v[ii] = r[ii * kD];
      tmem_st32(tm + kCbTmS + lane_off + q * 32, v);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();  // R_g (and at the first step R_0) fully read from shared memory
    if (tid == 0) {
      tc_fence_after();
      if (g + 1 <= nsteps) load_r(rs ^ 1, g + 1);  // the other stage held R_{g-1}, read by now
      wait_or_flag(&bar_m[s], (step >> 1) & 1, hdr, 41);
      const uint64_t b0 = desc_sw128(smem_u32(m_img(s)), 16, 1024);
#pragma unroll
      for (int k = 0; k < kD / 16; ++k)  // K-major B: +32 B per step inside a 64-wide block, +16 KiB per block
        mma_bf16_ts(tm + kCbTmS, tm + kCbTmA + k * 8, b0 + (uint64_t)(((k / 4) * 16384 + (k % 4) * 32) >> 4), idesc, 1);
      mma_commit(&bar_mma);
    }
    wait_or_flag(&bar_mma, step & 1, hdr, 42);
    tc_fence_after();
    if (tid == 0 && step + 2 < nsteps) load_m(s, g + 2);  // stage s is free: bring M_{g+2}
    // S_{g+1}: to the scan buffer and, as bf16, into the next A operand
#pragma unroll
    for (int q = 0; q < kD / 32; ++q) {
      float v[32];
      tmem_ld32(tm + kCbTmS + lane_off + q * 32, v);
#pragma unroll
      for (int ii = 0; ii < 32; ++ii) sb[(size_t)(g + 1) * kSt + (size_t)(q * 32 + ii) * kD + n] = v[ii];
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) pk[e] = pack2(v[2 * e], v[2 * e + 1]);
      tmem_st16u(tm + kCbTmA + lane_off + q * 16, pk);
    }
  }
  tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem_base, 256);
}

// =============================================== bounded-wait self-test
// Waits on an mbarrier that nothing ever completes, with a short limit, and
// reports the give-up exactly as the prefill kernels do (error word in the
// workspace header).  It lets a test exercise the failure path without
// faulting or hanging the GPU.
__global__ void kda_wait_selftest_kernel(WorkspaceHeader* hdr, uint32_t limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, limit)) {
    atomicOr(&hdr->error, 1u);
    atomicExch(&hdr->where, 99u);
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_arrive(&bar);  // leave the barrier completed
}

// ================================================================== host
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
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

// [B, T, H, 128] bf16 viewed as a 4-D tensor (channel, head, token, batch);
// box = 64 channels x 1 head x 64 tokens, 128-byte swizzle; tokens past T
// read as zeros.
// With d = 64 the box at channel 64 lies wholly outside the tensor and reads
// as zeros: the kernels then run on 128 channels of which the last 64 are
// zero (a zero key, query or value channel and a zero log-gate add nothing).
bool make_map(CUtensorMap* map, const void* base, int B, int T, int H, int d, bool swizzle = true) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_wait_selftest(void* ws, cudaStream_t stream) {
  WorkspaceHeader* hdr = static_cast<WorkspaceHeader*>(ws);
  cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(WorkspaceHeader), stream);
  if (e != cudaSuccess) return e;
  kda_wait_selftest_kernel<<<1, 32, 0, stream>>>(hdr, 1u << 12);
  return cudaGetLastError();
}

// Groups of the chunk-parallel scan for B*H chains of NC chunks (1 = no scan).
// Phase 3 runs G CTAs per chain, one per SM of a 148-SM part; phase 1 runs
// 2G-3 lighter CTAs per chain (two fit an SM).  The count is a fixed function
// of the shape so results do not depend on the GPU.
constexpr int kScanSMs = 148;
constexpr int kScanMinChunks = 4;
// With long chains (at least kScanLongChunks chunks per group at one phase-1
// CTA per SM) the group count is as large as the light phase-1 CTAs allow
// (two per SM, phase 3 still one wave): every group is shorter, which is what
// the sequential passes cost.  Otherwise more groups only add combination
// steps and launches (measured: 134 vs 77 us of state passes at B1 H16
// T4096 with 8 groups of 8 chunks instead of 6 of 11).
constexpr int kScanLongChunks = 256;
// Long chains whose final state does not overwrite the initial state also run
// the output pass of group 0 (which needs nothing from the scan) beside the
// light offset/transition passes, on the SMs those leave free: one more group
// then fits, with the other G - 1 output passes still one wave.
void scan_groups(int BH, int NC, int* G_out, int* L_out, bool* light = nullptr, bool early0 = false) {
  int G = 1;
  bool lt = false;
  if (BH > 0 && 3 * BH <= kScanSMs) {
    G = std::min((kScanSMs / BH + 3) / 2, NC / kScanMinChunks);
    if (G >= 3 && NC / G >= kScanLongChunks) {
      G = early0 ? std::min(kScanSMs / BH + 1, (2 * (kScanSMs - BH) / BH + 3) / 2)
                 : std::min(kScanSMs / BH, (2 * kScanSMs / BH + 3) / 2);
      G = std::min(G, NC / kScanMinChunks);
      lt = true;
    }
  }
  if (light) *light = lt;
  if (G >= 3) {
    const int L = (NC + G - 1) / G;
    G = (NC + L - 1) / L;
    if (G >= 3) {
      *G_out = G;
      *L_out = L;
      return;
    }
  }
  *G_out = 1;
  *L_out = NC;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the one before it in the stream still runs, and waits for it on the
// device (grid_dep_wait) before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

size_t prefill_bf16_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk) {
  (void)dk, (void)dv, (void)chunk;
  const int NC = (int)(((size_t)T + kC - 1) / kC);
  int G, L;
  scan_groups(B * H, NC, &G, &L);
  int G2, L2;
  scan_groups(B * H, NC, &G2, &L2, nullptr, true);  // the schedule with group 0's outputs early
  G = std::max(G, G2);
  const size_t scan = G > 1 ? 3 * (size_t)B * H * G * kD * kD * sizeof(float) : 0;
  return sizeof(WorkspaceHeader) + (size_t)B * H * NC * kRecBytes + scan;
}

// The preparation kernel in its backward mode (bf16, d_k = d_v = 128): the
// per-chunk operands of the backward's tensor-core state passes and local
// kernels for the (sequence, head) pairs out.bh0 .. out.bh0 + out.nbh - 1.
cudaError_t launch_prep_for_backward(const bf16* q, const bf16* k, const bf16* v, const bf16* g, const bf16* beta,
                                     float scale, int B, int T, int H, int gate, const PrepBwdOut& out,
                                     WorkspaceHeader* hdr, cudaStream_t stream) {
  static std::atomic<unsigned long long> attrs_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long dev_bit = dev < 64 ? 1ull << dev : 0ull;
  if (!(attrs_done.load(std::memory_order_acquire) & dev_bit) || !dev_bit) {
    for (auto kern : {kda_chunk_prep_kernel<false, false, true>, kda_chunk_prep_kernel<true, false, true>}) {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kP1Bytes + 1024);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
    }
    attrs_done.fetch_or(dev_bit, std::memory_order_release);
  }
  CUtensorMap mq, mk, mv, mg;
  memset(&mg, 0, sizeof(mg));
  if (!make_map(&mq, q, B, T, H, kD) || !make_map(&mk, k, B, T, H, kD) || !make_map(&mv, v, B, T, H, kD) ||
      (gate == KDA_GATE_CHANNEL && !make_map(&mg, g, B, T, H, kD)))
    return cudaErrorInvalidValue;
  const int NC = (T + kC - 1) / kC;
  const unsigned tiles = (unsigned)((size_t)out.nbh * NC);
  if (gate == KDA_GATE_CHANNEL)
    kda_chunk_prep_kernel<false, false, true><<<tiles, kP1Threads, kP1Bytes + 1024, stream>>>(
        mq, mk, mv, mg, beta, scale, nullptr, hdr, T, H, NC, nullptr, 0, out);
  else
    kda_chunk_prep_kernel<true, false, true><<<tiles, kP1Threads, kP1Bytes + 1024, stream>>>(
        mq, mk, mv, mg, beta, scale, nullptr, hdr, T, H, NC, gate == KDA_GATE_HEAD ? g : nullptr, 0, out);
  return cudaGetLastError();
}

int prefill_bf16_launches(int B, int T, int H) {
  const int NC = (int)(((size_t)T + kC - 1) / kC);
  int G, L;
  bool light = false;
  scan_groups(B * H, NC, &G, &L, &light, true);
  if (G == 1) return 2;
  // long chains: prep, group 0's output pass, offset/transition passes,
  // combination, the other output passes (4 launches when the final state
  // overwrites the initial state: group 0's outputs then follow the scan)
  return light ? 5 : 4;
}

cudaError_t launch_prefill_bf16(const bf16* q, const bf16* k, const bf16* v, const bf16* g, const bf16* beta,
                                float scale, const float* s0, bf16* o, float* sT, int B, int T, int H, int dk,
                                int dv, int chunk, int gate, int prep, void* ws, size_t ws_bytes,
                                cudaStream_t stream, void* const* events) {
  (void)chunk, (void)ws_bytes;
  // Function attributes belong to each device's context: set them once per
  // device (one bit per device ordinal; ordinals past 63 set them every call).
  static std::atomic<unsigned long long> attrs_done{0};
  int dev = 0;
  const cudaError_t dev_err = cudaGetDevice(&dev);
  if (dev_err != cudaSuccess) return dev_err;
  const unsigned long long dev_bit = dev < 64 ? 1ull << dev : 0ull;
  if (!(attrs_done.load(std::memory_order_acquire) & dev_bit) || !dev_bit) {
    for (auto kern : {kda_chunk_prep_kernel<false, false>, kda_chunk_prep_kernel<true, false>,
                      kda_chunk_prep_kernel<false, true>, kda_chunk_prep_kernel<true, true>}) {
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kP1Bytes + 1024);
      if (e != cudaSuccess) return e;
      // kP1Blocks CTAs per SM need nearly all of the SM's shared memory
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
    }
    cudaError_t e;
    e = cudaFuncSetAttribute(kda_state_pass_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kP2Bytes + 1024);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_state_pass_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kP2BytesNoOut + 1024);
    if (e != cudaSuccess) return e;
    // two of them share an SM
    e = cudaFuncSetAttribute(kda_state_pass_kernel<false>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_scan_combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCbSmem);
    if (e != cudaSuccess) return e;
    attrs_done.fetch_or(dev_bit, std::memory_order_release);
  }
  CUtensorMap mq, mk, mv, mg, mo;
  memset(&mg, 0, sizeof(mg));  // only the per-channel gate is read through a tensor map
  if (!make_map(&mq, q, B, T, H, dk) || !make_map(&mk, k, B, T, H, dk) || !make_map(&mv, v, B, T, H, dv) ||
      (gate == KDA_GATE_CHANNEL && !make_map(&mg, g, B, T, H, dk)) || !make_map(&mo, o, B, T, H, dv, false))
    return cudaErrorInvalidValue;
  const int NC = (T + kC - 1) / kC;
  WorkspaceHeader* hdr = static_cast<WorkspaceHeader*>(ws);
  uint8_t* records = static_cast<uint8_t*>(ws) + sizeof(WorkspaceHeader);
  cudaError_t e = mark(events, 0, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(hdr, 0, sizeof(WorkspaceHeader), stream);
  if (e != cudaSuccess) return e;
  const unsigned tiles = (unsigned)((size_t)B * H * NC);
  {
    const bool scalar = gate != KDA_GATE_CHANNEL;
    const bf16* gh = gate == KDA_GATE_HEAD ? g : nullptr;
    auto kern = scalar ? (prep ? kda_chunk_prep_kernel<true, true> : kda_chunk_prep_kernel<true, false>)
                       : (prep ? kda_chunk_prep_kernel<false, true> : kda_chunk_prep_kernel<false, false>);
    kern<<<tiles, kP1Threads, kP1Bytes + 1024, stream>>>(mq, mk, mv, mg, beta, scale, records, hdr, T, H, NC, gh, prep,
                                                         PrepBwdOut{});
  }
  e = cudaGetLastError();
  if (e == cudaSuccess) e = mark(events, 1, stream);
  if (e != cudaSuccess) return e;
  StatePassArgs a{records, hdr, s0, sT, nullptr, nullptr, nullptr, T, H, NC, 1, NC, 0, dk, dv, 0, 0, 0, 1, 0};
  const int BH = B * H;
  int G, L;
  bool light = false;
  const bool in_place = s0 != nullptr && (const void*)s0 == (const void*)sT;
  scan_groups(BH, NC, &G, &L, &light, !in_place);
  const bool early0 = light && !in_place && G > 1;
  if (G == 1) {
    e = launch_dependent(kda_state_pass_kernel<true>, (unsigned)BH, kSPThreads, kP2Bytes + 1024, stream, mo, a);
  } else {
    float* scan = reinterpret_cast<float*>(records + (size_t)BH * NC * kRecBytes);
    const size_t per = (size_t)BH * G * kD * kD;
    a.rbuf = scan;
    a.mbuf = scan + per;
    a.sbuf = scan + 2 * per;
    a.G = G;
    a.L = L;
    if (early0) {
      // group 0's output pass first, launched in plain stream order (with a
      // programmatic launch its CTAs took SMs in the prep's last wave and
      // waited there: 31.8 vs 30.9 ms per call at T = 1,048,576); it lets the
      // offset/transition passes be scheduled beside it, and those need no
      // wait (the prep had finished before this grid started)
      a.phase = 3;
      a.g_first = 0, a.g_count = 1, a.s0_direct = 1, a.trigger = 1;
      kda_state_pass_kernel<true><<<(unsigned)BH, kSPThreads, kP2Bytes + 1024, stream>>>(mo, a);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      a.g_count = 0, a.s0_direct = 0, a.trigger = 0, a.dep_wait = 0;
    }
    a.phase = 1;
    e = light ? launch_dependent(kda_state_pass_kernel<false>, (unsigned)(BH * (2 * G - 3)), kSPThreadsNoOut,
                                 kP2BytesNoOut + 1024, stream, mo, a)
              : launch_dependent(kda_state_pass_kernel<true>, (unsigned)(BH * (2 * G - 3)), kSPThreads,
                                 kP2Bytes + 1024, stream, mo, a);
    if (e != cudaSuccess) return e;
    a.dep_wait = 1;
    e = launch_dependent(kda_scan_combine_kernel, (unsigned)BH, kCbThreads, kCbSmem, stream, scan + 2 * per,
                         (const float*)scan, (const float*)(scan + per), G, hdr);
    if (e != cudaSuccess) return e;
    a.phase = 3;
    if (early0) a.g_first = 1, a.g_count = G - 1;
    e = launch_dependent(kda_state_pass_kernel<true>, (unsigned)(BH * (early0 ? G - 1 : G)), kSPThreads,
                         kP2Bytes + 1024, stream, mo, a);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e == cudaSuccess) e = mark(events, 2, stream);
  return e;
}

}  // namespace kda
