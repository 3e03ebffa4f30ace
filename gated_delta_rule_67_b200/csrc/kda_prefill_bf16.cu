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
// Two kernels:
//  1. kda_chunk_prep: one CTA per (sequence, head, chunk), fully parallel.
//     TMA brings q, k, v, g (64 x 128 bf16 tiles, 128-byte swizzle); the CTA
//     computes G and the decayed operands, the two score matrices with one
//     tcgen05 MMA (M=128: rows 0-63 give A_kk, rows 64-127 give A_qk), the
//     triangular inverse on the CUDA cores in fp32, and W^T, U^T with two
//     more MMAs.  It writes, per chunk, a record of ready-to-use operand
//     images (already in the swizzled shared-memory layout the MMA reads):
//     [-W ; Q+] (128 x 128), A_qk (64 x 64), Kbar (64 x 128), U (64 x 128
//     plain) and gamma = exp(G_C) (128 fp32).
//  2. kda_state_pass: one CTA per (sequence, head); walks the chunks in
//     order with the state S^T (d_v x d_k, fp32) resident in tensor memory.
//     Per chunk: S0^T -> bf16 operand, S <- gamma*S in place; one MMA gives
//     [-S0^T W^T | S0^T Q+^T]; V'^T = U^T + first half; then O^T += V'^T A_qk^T
//     and S^T += V'^T Kbar.  The next chunk's record is prefetched with a
//     bulk copy while the current one is processed.
//
// Everything is transposed relative to the token-major notation above so
// that every MMA has M = 128 (the d_v or d_k dimension) and each TMEM lane is
// one channel.
#include <cudaTypedefs.h>

#include "kda_common.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;
using bf16 = __nv_bfloat16;

constexpr int kC = 64;    // chunk length
constexpr int kD = 128;   // d_k = d_v
constexpr int kRefTok = 31;

// --- per-chunk record in the workspace (byte offsets) -----------------------
constexpr uint32_t kRecWQ = 0;          // [-W ; Q+]: K-major, 128 rows x 128 ch (32 KiB)
constexpr uint32_t kRecAqk = 32768;     // A_qk: K-major, 64 rows (i) x 64 (j)  (8 KiB)
constexpr uint32_t kRecKbar = 40960;    // Kbar: token-row 128B-swizzled tile 64 x 128 (16 KiB)
constexpr uint32_t kRecU = 57344;       // U: plain row-major [64][128] bf16 (16 KiB)
constexpr uint32_t kRecGamma = 73728;   // gamma: 128 fp32
constexpr uint32_t kRecBytes = 74240;

// --- prep kernel shared memory (byte offsets from a 1024-aligned base) -----
constexpr uint32_t kP1Q = 0;            // q tile (token rows), 16 KiB
constexpr uint32_t kP1K = 16384;        // k tile, overwritten in place by K+ (start-decayed)
constexpr uint32_t kP1V = 32768;        // v tile
constexpr uint32_t kP1G = 49152;        // g tile; dead after the cumulative sum
constexpr uint32_t kP1A1 = 49152;       // score A operand [K+_r ; Q+_r], 128 rows, 32 KiB (aliases g)
constexpr uint32_t kP1Akk = 49152;      // fp32 A_kk [64][kAkkLd] for the solve (aliases A1)
constexpr uint32_t kP1B1 = 81920;       // score B operand K-_r, 64 rows, 16 KiB
constexpr uint32_t kP1B2 = 81920;       // (T diag beta)^T operand, 64 x 64, 8 KiB (aliases B1)
constexpr uint32_t kP1Bytes = 98304;
constexpr int kAkkLd = 68;              // padded fp32 row stride of A_kk

// --- state-pass kernel shared memory --------------------------------------
constexpr uint32_t kStage = 74752;      // record rounded up to 1024
constexpr uint32_t kP2S = 2 * kStage;   // S0^T bf16, K-major 128 rows x 128 (32 KiB)
constexpr uint32_t kP2Vp = kP2S + 32768;// V'^T bf16, K-major 128 rows x 64 (16 KiB)
constexpr uint32_t kP2Bytes = kP2Vp + 16384;

constexpr uint32_t kWaitLimit = 1u << 24;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ float ldbf(const uint8_t* base, uint32_t off) {
  return __bfloat162float(*reinterpret_cast<const bf16*>(base + off));
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

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int32_t x, int32_t y,
                                            int32_t z, int32_t w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void wait_or_flag(uint64_t* bar, uint32_t parity, WorkspaceHeader* hdr, uint32_t where) {
  if (!mbar_wait(bar, parity, kWaitLimit)) {
    atomicOr(&hdr->error, 1u);
    atomicExch(&hdr->where, where);
  }
}

// =============================================================== kernel 1
__global__ void __launch_bounds__(128, 2)
    kda_chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                          const bf16* __restrict__ beta, float scale, uint8_t* __restrict__ records,
                          WorkspaceHeader* hdr, int T, int H, int NC) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ uint64_t bar_tma, bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ float sbeta[kC];

  const int tid = threadIdx.x, warp = tid >> 5;
  const int chunk = blockIdx.x % NC;
  const int bh = blockIdx.x / NC;
  const int h = bh % H, b = bh / H;
  const int t0 = chunk * kC;
  const int L = min(kC, T - t0);
  uint8_t* rec = records + (size_t)blockIdx.x * kRecBytes;

  if (tid == 0) {
    mbar_init(&bar_tma, 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base, 256);
  if (tid < kC) sbeta[tid] = tid < L ? __bfloat162float(beta[((size_t)b * T + t0 + tid) * H + h]) : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tmem_base;

  if (tid == 0) {
    mbar_expect_tx(&bar_tma, 4 * 16384);
    const CUtensorMap* maps[4] = {&tm_q, &tm_k, &tm_v, &tm_g};
    const uint32_t dst[4] = {kP1Q, kP1K, kP1V, kP1G};
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      tma_load_4d(sm + dst[m], maps[m], &bar_tma, 0, h, t0, b);
      tma_load_4d(sm + dst[m] + 8192, maps[m], &bar_tma, 64, h, t0, b);
    }
  }
  wait_or_flag(&bar_tma, 0, hdr, 1);

  // ---- pass 1: in-chunk cumulative log-gate, one key channel per thread
  const int ch = tid;
  float G[kC];
  {
    float run = 0.f;
#pragma unroll
    for (int i = 0; i < kC; ++i) {
      run += ldbf(sm + kP1G, kmajor_off(i, ch, kC));
      G[i] = run;
    }
  }
  __syncthreads();  // the g tile is dead from here on (A1 aliases it)

  // ---- pass 2: decayed operands
  {
    const float gref = G[kRefTok], gend = G[kC - 1];
#pragma unroll
    for (int i = 0; i < kC; ++i) {
      const uint32_t o64 = kmajor_off(i, ch, kC);
      const float kk = ldbf(sm + kP1K, o64);
      const float qq = ldbf(sm + kP1Q, o64);
      const float em = __expf(G[i] - gref);
      const float ei = __expf(gref - G[i]);
      const float e0 = __expf(G[i]);
      const float eb = __expf(gend - G[i]);
      stbf(sm + kP1A1, kmajor_off(i, ch, 128), kk * em);                 // K+_r
      stbf(sm + kP1A1, kmajor_off(kC + i, ch, 128), scale * qq * em);    // Q+_r
      stbf(sm + kP1B1, o64, kk * ei);                                    // K-_r
      stbf(sm + kP1K, o64, kk * e0);                                     // K+ (chunk start), in place
      stbf(rec + kRecWQ, kmajor_off(kC + i, ch, 128), scale * qq * e0);  // Q+ image rows 64..127
      stbf(rec + kRecKbar, o64, kk * eb);                                // Kbar image
    }
    reinterpret_cast<float*>(rec + kRecGamma)[ch] = expf(gend);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- score MMA: D[0:128, 0:64] = [K+_r ; Q+_r] (128 x 128) . K-_r^T
  if (tid == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
    const uint32_t a0 = smem_u32(sm + kP1A1), b0 = smem_u32(sm + kP1B1);
#pragma unroll
    for (int s = 0; s < kD / 16; ++s) {
      const uint32_t a = a0 + (s / 4) * 16384 + (s % 4) * 32;
      const uint32_t bb = b0 + (s / 4) * 8192 + (s % 4) * 32;
      mma_bf16(tm, desc_sw128(a, 16, 1024), desc_sw128(bb, 16, 1024), idesc, s > 0);
    }
    mma_commit(&bar_mma);
  }
  wait_or_flag(&bar_mma, 0, hdr, 2);
  tc_fence_after();

  // ---- masks: rows 0..63 -> A_kk (fp32, smem), rows 64..127 -> A_qk image
  {
    float* akk = reinterpret_cast<float*>(sm + kP1Akk);
    const int r = tid & 63;
#pragma unroll
    for (int cb = 0; cb < kC / 16; ++cb) {
      float v[16];
      tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + cb * 16, v);
      tmem_wait_ld();
      if (warp < 2) {
        const float br = sbeta[r];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int j = cb * 16 + jj;
          akk[r * kAkkLd + j] = j < r ? br * v[jj] : 0.f;
        }
      } else {
        float m[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) m[jj] = (cb * 16 + jj) <= r ? v[jj] : 0.f;
        st_kmajor8(rec + kRecAqk, r, cb * 16, kC, m);
        st_kmajor8(rec + kRecAqk, r, cb * 16 + 8, kC, m + 8);
      }
    }
  }
  __syncthreads();

  // ---- T = (I + A_kk)^-1, one column per thread (threads 0..63), fp32
  if (tid < kC) {
    const int j = tid;
    const float* akk = reinterpret_cast<const float*>(sm + kP1Akk);
    float t[kC];
#pragma unroll
    for (int i = 0; i < kC; ++i) {
      float acc0 = 0.f, acc1 = 0.f;
      const float4* row = reinterpret_cast<const float4*>(akk + i * kAkkLd);
#pragma unroll
      for (int m4 = 0; m4 < i / 4; ++m4) {
        const float4 a = row[m4];
        acc0 = fmaf(a.x, t[4 * m4 + 0], acc0);
        acc1 = fmaf(a.y, t[4 * m4 + 1], acc1);
        acc0 = fmaf(a.z, t[4 * m4 + 2], acc0);
        acc1 = fmaf(a.w, t[4 * m4 + 3], acc1);
      }
#pragma unroll
      for (int m = (i / 4) * 4; m < i; ++m) acc0 = fmaf(akk[i * kAkkLd + m], t[m], acc0);
      t[i] = i < j ? 0.f : (i == j ? 1.f : -(acc0 + acc1));
    }
    // (T diag(beta))^T as the K-major B operand: row n = i, column k = j.
    const float bj = sbeta[j];
#pragma unroll
    for (int i = 0; i < kC; ++i) stbf(sm + kP1B2, kmajor_off(i, j, kC), t[i] * bj);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- W^T = K+^T (T diag beta)^T and U^T = V^T (T diag beta)^T  (M=128, N=64, K=64)
  if (tid == 0) {
    const uint32_t idesc = idesc_bf16_f32(128, 64, 1, 0);
    const uint32_t kb = smem_u32(sm + kP1K), vb = smem_u32(sm + kP1V), b2 = smem_u32(sm + kP1B2);
#pragma unroll
    for (int s = 0; s < kC / 16; ++s) {
      const uint64_t bd = desc_sw128(b2 + s * 32, 16, 1024);
      mma_bf16(tm + 64, desc_sw128(kb + 2 * s * 1024, 8192, 1024), bd, idesc, s > 0);
      mma_bf16(tm + 128, desc_sw128(vb + 2 * s * 1024, 8192, 1024), bd, idesc, s > 0);
    }
    mma_commit(&bar_mma);
  }
  wait_or_flag(&bar_mma, 1, hdr, 3);
  tc_fence_after();

  // ---- -W into rows 0..63 of the [-W ; Q+] image, U as plain rows
  {
    const int c = tid;
    bf16* uimg = reinterpret_cast<bf16*>(rec + kRecU);
#pragma unroll
    for (int cb = 0; cb < kC / 16; ++cb) {
      float w[16], u[16];
      tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + 64 + cb * 16, w);
      tmem_ld16(tm + ((uint32_t)(warp * 32) << 16) + 128 + cb * 16, u);
      tmem_wait_ld();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int i = cb * 16 + ii;
        stbf(rec + kRecWQ, kmajor_off(i, c, 128), -w[ii]);
        uimg[i * kD + c] = __float2bfloat16_rn(u[ii]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 256);
}

// =============================================================== kernel 2
__global__ void __launch_bounds__(128, 1)
    kda_state_pass_kernel(const uint8_t* __restrict__ records, WorkspaceHeader* hdr, const float* s0, float* sT,
                          bf16* __restrict__ o, int T, int H, int NC) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ uint64_t bar_full[2], bar_mma;
  __shared__ uint32_t tmem_base;

  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = blockIdx.x;
  const int h = bh % H, b = bh / H;
  const uint8_t* recs = records + (size_t)bh * NC * kRecBytes;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  if (tid == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&tmem_base, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tS = tmem_base, tD = tmem_base + 128;

  if (tid == 0) {
    mbar_expect_tx(&bar_full[0], kRecBytes);
    bulk_load(sm, recs, kRecBytes, &bar_full[0]);
  }
  // S^T row j (= column j of S) into TMEM lane j.
  const int j = tid;
  const size_t sbase = (size_t)bh * kD * kD;
#pragma unroll
  for (int cb = 0; cb < kD / 16; ++cb) {
    float v[16];
#pragma unroll
    for (int ii = 0; ii < 16; ++ii) v[ii] = s0 ? s0[sbase + (size_t)(cb * 16 + ii) * kD + j] : 0.f;
    tmem_st16(tS + lane_off + cb * 16, v);
  }
  tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  uint32_t mma_phase = 0;
  for (int n = 0; n < NC; ++n) {
    const int st = n & 1;
    uint8_t* stage = sm + st * kStage;
    if (tid == 0 && n + 1 < NC) {
      mbar_expect_tx(&bar_full[st ^ 1], kRecBytes);
      bulk_load(sm + (st ^ 1) * kStage, recs + (size_t)(n + 1) * kRecBytes, kRecBytes, &bar_full[st ^ 1]);
    }
    wait_or_flag(&bar_full[st], (n >> 1) & 1, hdr, 10);

    // (A) S0^T -> bf16 operand; S^T <- S^T Diag(gamma) in place
    {
      const float* gam = reinterpret_cast<const float*>(stage + kRecGamma);
#pragma unroll
      for (int cb = 0; cb < kD / 16; ++cb) {
        float v[16];
        tmem_ld16(tS + lane_off + cb * 16, v);
        tmem_wait_ld();
        st_kmajor8(sm + kP2S, j, cb * 16, kD, v);
        st_kmajor8(sm + kP2S, j, cb * 16 + 8, kD, v + 8);
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) v[ii] *= gam[cb * 16 + ii];
        tmem_st16(tS + lane_off + cb * 16, v);
      }
      tmem_wait_st();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // (B) D = S0^T [-W ; Q+]^T : cols 0..63 = -(W S0)^T, cols 64..127 = (Q+ S0)^T
    if (tid == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t a0 = smem_u32(sm + kP2S), b0 = smem_u32(stage + kRecWQ);
#pragma unroll
      for (int s = 0; s < kD / 16; ++s) {
        const uint32_t off = (s / 4) * 16384 + (s % 4) * 32;
        mma_bf16(tD, desc_sw128(a0 + off, 16, 1024), desc_sw128(b0 + off, 16, 1024), idesc, s > 0);
      }
      mma_commit(&bar_mma);
    }
    wait_or_flag(&bar_mma, mma_phase, hdr, 11);
    mma_phase ^= 1;
    tc_fence_after();

    // (C) V'^T = U^T - (W S0)^T -> bf16 operand
    {
      const bf16* u = reinterpret_cast<const bf16*>(stage + kRecU);
#pragma unroll
      for (int cb = 0; cb < kC / 16; ++cb) {
        float v[16];
        tmem_ld16(tD + lane_off + cb * 16, v);
        tmem_wait_ld();
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) v[ii] += __bfloat162float(u[(cb * 16 + ii) * kD + j]);
        st_kmajor8(sm + kP2Vp, j, cb * 16, kD, v);
        st_kmajor8(sm + kP2Vp, j, cb * 16 + 8, kD, v + 8);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // (D) O^T += V'^T A_qk^T ;  S^T += V'^T Kbar
    if (tid == 0) {
      const uint32_t id_o = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t id_s = idesc_bf16_f32(128, 128, 0, 1);
      const uint32_t vp = smem_u32(sm + kP2Vp), aq = smem_u32(stage + kRecAqk), kbar = smem_u32(stage + kRecKbar);
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint64_t ad = desc_sw128(vp + s * 32, 16, 1024);
        mma_bf16(tD + 64, ad, desc_sw128(aq + s * 32, 16, 1024), id_o, 1);
        mma_bf16(tS, ad, desc_sw128(kbar + 2 * s * 1024, 8192, 1024), id_s, 1);
      }
      mma_commit(&bar_mma);
    }
    wait_or_flag(&bar_mma, mma_phase, hdr, 12);
    mma_phase ^= 1;
    tc_fence_after();

    // (E) output rows of this chunk
    {
      const int t0 = n * kC;
      const int L = min(kC, T - t0);
      bf16* orow = o + (((size_t)b * T + t0) * H + h) * kD + j;
#pragma unroll
      for (int cb = 0; cb < kC / 16; ++cb) {
        float v[16];
        tmem_ld16(tD + lane_off + 64 + cb * 16, v);
        tmem_wait_ld();
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          const int i = cb * 16 + ii;
          if (i < L) orow[(size_t)i * H * kD] = __float2bfloat16_rn(v[ii]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (sT) {
#pragma unroll
    for (int cb = 0; cb < kD / 16; ++cb) {
      float v[16];
      tmem_ld16(tS + lane_off + cb * 16, v);
      tmem_wait_ld();
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) sT[sbase + (size_t)(cb * 16 + ii) * kD + j] = v[ii];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem_base, 256);
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
bool make_map(CUtensorMap* map, const void* base, int B, int T, int H) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)kD * 2, (cuuint64_t)H * kD * 2, (cuuint64_t)T * H * kD * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)kC, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_bf16_workspace_bytes(int B, int T, int H, int dk, int dv, int chunk) {
  (void)dk, (void)dv, (void)chunk;
  const size_t nc = ((size_t)T + kC - 1) / kC;
  return sizeof(WorkspaceHeader) + (size_t)B * H * nc * kRecBytes;
}

cudaError_t launch_prefill_bf16(const bf16* q, const bf16* k, const bf16* v, const bf16* g, const bf16* beta,
                                float scale, const float* s0, bf16* o, float* sT, int B, int T, int H, int dk,
                                int dv, int chunk, void* ws, size_t ws_bytes, cudaStream_t stream,
                                void* const* events) {
  (void)dk, (void)dv, (void)chunk, (void)ws_bytes;
  static bool attrs_set = false;
  if (!attrs_set) {
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kP1Bytes + 1024);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_state_pass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kP2Bytes + 1024);
    if (e != cudaSuccess) return e;
    attrs_set = true;
  }
  CUtensorMap mq, mk, mv, mg;
  if (!make_map(&mq, q, B, T, H) || !make_map(&mk, k, B, T, H) || !make_map(&mv, v, B, T, H) ||
      !make_map(&mg, g, B, T, H))
    return cudaErrorInvalidValue;
  const int NC = (T + kC - 1) / kC;
  WorkspaceHeader* hdr = static_cast<WorkspaceHeader*>(ws);
  uint8_t* records = static_cast<uint8_t*>(ws) + sizeof(WorkspaceHeader);
  cudaError_t e = mark(events, 0, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(hdr, 0, sizeof(WorkspaceHeader), stream);
  if (e != cudaSuccess) return e;
  const unsigned tiles = (unsigned)((size_t)B * H * NC);
  kda_chunk_prep_kernel<<<tiles, 128, kP1Bytes + 1024, stream>>>(mq, mk, mv, mg, beta, scale, records, hdr, T, H,
                                                                  NC);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = mark(events, 1, stream);
  if (e != cudaSuccess) return e;
  kda_state_pass_kernel<<<(unsigned)(B * H), 128, kP2Bytes + 1024, stream>>>(records, hdr, s0, sT, o, T, H, NC);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = mark(events, 2, stream);
  return e;
}

}  // namespace kda
