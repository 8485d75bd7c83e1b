// kda_chunk_tc.cuh -- chunkwise-parallel KDA prefill on sm_100a tensor cores.
//
// The pages ("Kimi Linear" summary, section "Algoritmo paralelo por chunks")
// state the shape of the method: fixed-size chunks, the final state of one
// chunk seeds the next, a WY / UT representation of the chunk's rank-1 updates
// built with a lower-triangular inverse (forward substitution), and an output
// that adds an inter-chunk recurrent term to an intra-chunk parallel term,
// organised as matrix products for the tensor cores.  The algebra below is
// derived from the recurrence
//     S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1} + b_t k_t v_t^T,  o_t = S_t^T q_t.
//
// Within a chunk of C = 64 tokens r (state S at the chunk start), with
// g_r = cumsum(log_alpha)_r per key channel, Gamma_r = exp(g_r),
// Psi_r = exp(g_last - g_r), gamma_C = exp(g_last):
//     A  = strict_tril( Diag(b) (K o Gamma)(K / Gamma)^T )       (C x C)
//     T  = (I + A)^-1,  Tb = T Diag(b)
//     W  = Tb (K o Gamma)          U' = Tb V        (pseudo-keys / -values)
//     U  = U' - W S                                  (the chunk's deltas)
//     P  = tril( (Q o Gamma)(K / Gamma)^T )           (diagonal included)
//     O  = (Q o Gamma) S + P U
//     S' = Diag(gamma_C) S + (K o Psi)^T U
// The products (K o Gamma)(K/Gamma)^T are formed with a per-channel reference
// point ref_c = g_last/2, i.e. (K o e^{g-ref})(K o e^{ref-g})^T, so no factor
// leaves [e^-80, e^80] while the chunk's total decay is at most 160 nats (the
// pages' warning that fine-grained decay makes intra-chunk divisions
// imprecise, section "Menos computacao que o DPLR geral").  Chunks that decay
// more take an exact CUDA-core path for A and P with exp(g_r - g_s) per term.
//
// Two kernels:
//   kda_chunk_prep_kernel  one CTA per (chunk, head), fully parallel: A and P
//       on tcgen05 (M=128 stacked [K;Q] x K^T), T by blocked forward
//       substitution on CUDA cores, W on tcgen05 (M=64), and every operand the
//       recurrence needs, written to the workspace as a 82,432-byte slot in
//       the exact K-major core-matrix layout the MMA descriptors read.
//   kda_chunk_rec_kernel   one CTA per (sequence, head): walks the chunks in
//       order.  A producer warp streams slots into a 2-deep shared-memory ring
//       with bulk async copies; one thread issues the tcgen05 MMAs
//         U^T  = [V^T | S^T] x [Tb | -W]^T        (M=128 v, N=64, K=64+128)
//         O1^T = S^T x (Q o Gamma)^T              (M=128, N=64, K=128)
//         dS^T = U^T x (K o Psi)                  (M=128, N=128, K=64)
//         O^T += U^T x P^T                        (M=128, N=64, K=64)
//       and eight warps (one TMEM lane = one value column v each) keep the
//       fp32 state S^T in registers, apply S <- gamma_C S + dS and feed bf16
//       copies of S^T and U^T back as MMA operands.
#pragma once

#include "kda_ptx.cuh"

namespace kda {
namespace tc {

constexpr int C = 64;    // chunk length
constexpr int D = 128;   // dk = dv

// ---- workspace slot: MMA-ready operand tiles of one (chunk, head) ---------
constexpr uint32_t BU_OFF = 0;        // [64 r][192]  (Tb | -W), K-major
constexpr uint32_t BO_OFF = 24576;    // [64 r][128]  Q o Gamma
constexpr uint32_t BS_OFF = 40960;    // [128 c][64]  (K o Psi)^T
constexpr uint32_t BP_OFF = 57344;    // [64 r'][64]  P
constexpr uint32_t AV_OFF = 65536;    // [128 v][64]  V^T
constexpr uint32_t GC_OFF = 81920;    // float[128]   gamma_C
constexpr uint32_t SLOT_BYTES = 82432;

constexpr float kFastSpan = 160.0f;   // max total chunk decay (nats) of the fast path

// ---- prep kernel shared memory --------------------------------------------
constexpr int GST = 136;  // padded fp32 row stride of the cumsum tile
constexpr int AST = 65;   // padded row stride of A / T (fp32)
constexpr uint32_t P_SLOT = 0;
constexpr uint32_t P_KQA = SLOT_BYTES;            // [128][128] bf16: rows 0-63 K o e1, 64-127 Q o e1
constexpr uint32_t P_KB = P_KQA + 32768;          // [64][128]  K o e2
constexpr uint32_t P_KGT = P_KB + 16384;          // [128 c][64 s] (K o Gamma)^T
constexpr uint32_t P_G = P_KGT + 16384;           // fp32 [64][GST]
constexpr uint32_t P_VEC = P_G + 64 * GST * 4;    // beta[64], ref[128], sc[128]
constexpr uint32_t P_BAR = P_VEC + (64 + 128 + 128) * 4;
constexpr uint32_t P_SMEM = P_BAR + 64;
// aliases of the KQA/KB region once the A/P product has been consumed
constexpr uint32_t P_AF = P_KQA;                  // fp32 [64][AST]  A
constexpr uint32_t P_TF = P_AF + 64 * AST * 4;    // fp32 [64][AST]  T
constexpr uint32_t P_X = P_TF + 64 * AST * 4;     // fp32 [3][16][17] scratch
static_assert(P_X + 3 * 16 * 17 * 4 <= P_KGT, "A/T scratch must fit in the KQA/KB region");

// Locate chunk `g` of the flattened (sequence, chunk) list.
__device__ __forceinline__ bool find_chunk(int g, int N, int T, const int32_t* cu, int* n_out, int64_t* t0_out,
                                           int* len_out) {
  int base = 0;
  for (int n = 0; n < N; ++n) {
    const int64_t s = cu ? cu[n] : static_cast<int64_t>(n) * T;
    const int64_t e = cu ? cu[n + 1] : s + T;
    const int nc = static_cast<int>((e - s + C - 1) / C);
    if (g < base + nc) {
      const int j = g - base;
      *n_out = n;
      *t0_out = s + static_cast<int64_t>(j) * C;
      const int64_t rem = e - *t0_out;
      *len_out = rem < C ? static_cast<int>(rem) : C;
      return true;
    }
    base += nc;
  }
  return false;
}

__device__ __forceinline__ void st_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ float2 ld_pair(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

template <typename TG>
__device__ __forceinline__ float ld_gate(const TG* p);
template <>
__device__ __forceinline__ float ld_gate<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_gate<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// ===========================================================================
// prep: one CTA (256 threads) per (chunk g = blockIdx.x, head h = blockIdx.y)
// ===========================================================================
template <typename TG>
__global__ void __launch_bounds__(256, 1)
    kda_chunk_prep_kernel(int N, int T, int H, const int32_t* __restrict__ cu, const __nv_bfloat16* __restrict__ q,
                          const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                          const TG* __restrict__ la, const TG* __restrict__ beta, uint8_t* __restrict__ ws) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.x, h = blockIdx.y;
  int n, L;
  int64_t t0;
  if (!find_chunk(g, N, T, cu, &n, &t0, &L)) return;  // grid is an upper bound on the chunk count

  uint8_t* slot = smem + P_SLOT;
  float* G = reinterpret_cast<float*>(smem + P_G);
  float* sbeta = reinterpret_cast<float*>(smem + P_VEC);
  float* sref = sbeta + 64;
  float* ssc = sref + 128;
  uint64_t* bar_ap = reinterpret_cast<uint64_t*>(smem + P_BAR);
  uint64_t* bar_w = bar_ap + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_ap + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar_ap + 3);
  float* gC = reinterpret_cast<float*>(slot + GC_OFF);
  const uint32_t s_base = smem_u32(smem);

  if (tid == 0) {
    mbar_init(bar_ap, 1);
    mbar_init(bar_w, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }

  // ---- load log_alpha (fp32, rows >= L zero) and beta -----------------------
  for (int i = tid; i < 64 * 32; i += 256) {  // 64 rows x 32 groups of 4 channels
    const int r = i >> 5, c4 = (i & 31) * 4;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < L) {
      const TG* p = la + ((t0 + r) * H + h) * D + c4;
      x = make_float4(ld_gate(p), ld_gate(p + 1), ld_gate(p + 2), ld_gate(p + 3));
    }
    *reinterpret_cast<float4*>(G + r * GST + c4) = x;
  }
  if (tid < 64) sbeta[tid] = tid < L ? ld_gate(beta + (t0 + tid) * H + h) : 0.f;
  __syncthreads();

  // ---- cumulative log-decay per channel (two half scans) --------------------
  {
    const int c = tid & 127, half = tid >> 7;
    float x[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = G[(32 * half + i) * GST + c];
#pragma unroll
    for (int i = 1; i < 32; ++i) x[i] += x[i - 1];
    __syncthreads();
    if (half == 0) {
#pragma unroll
      for (int i = 0; i < 32; ++i) G[i * GST + c] = x[i];
    }
    __syncthreads();
    if (half == 1) {
      const float off = G[31 * GST + c];
#pragma unroll
      for (int i = 0; i < 32; ++i) G[(32 + i) * GST + c] = x[i] + off;
    }
    __syncthreads();
  }
  float glast = 0.f;
  if (tid < 128) {
    glast = G[63 * GST + tid];
    sref[tid] = 0.5f * glast;
    ssc[tid] = __expf(0.5f * glast);
    gC[tid] = __expf(glast);
  }
  const bool slow = __syncthreads_or(tid < 128 && -glast > kFastSpan) != 0;

  // ---- elementwise pass in stmatrix fragment layout --------------------------
  // warp w owns rows 8w..8w+7; lane t: row 8w + t/4, columns 32cb + 8b + 2(t%4) + {0,1}
  {
    const int rr = lane >> 2, cc = (lane & 3) * 2;
    const int r = 8 * warp + rr;
    const bool live = r < L;
    const int64_t grow = (t0 + r) * H + h;
    const uint32_t li = lane >> 3, lr = lane & 7;
    for (int cb = 0; cb < 4; ++cb) {
      uint32_t ka[4], qa[4], kb[4], qd[4], kg[4], kt[4], vv[4];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int c = 32 * cb + 8 * b + cc;
        float2 kx = make_float2(0.f, 0.f), qx = kx, vx = kx;
        if (live) {
          kx = ld_pair(k + grow * D + c);
          qx = ld_pair(q + grow * D + c);
          vx = ld_pair(v + grow * D + c);
        }
        const float2 gx = *reinterpret_cast<const float2*>(G + r * GST + c);
        float gam0, gam1, psi0, psi1;
        if (!slow) {
          const float e10 = __expf(gx.x - sref[c]), e11 = __expf(gx.y - sref[c + 1]);
          const float e20 = __expf(sref[c] - gx.x), e21 = __expf(sref[c + 1] - gx.y);
          ka[b] = pack_bf16(kx.x * e10, kx.y * e11);
          qa[b] = pack_bf16(qx.x * e10, qx.y * e11);
          kb[b] = pack_bf16(kx.x * e20, kx.y * e21);
          gam0 = ssc[c] * e10;
          gam1 = ssc[c + 1] * e11;
          psi0 = ssc[c] * e20;
          psi1 = ssc[c + 1] * e21;
        } else {
          const float gl0 = 2.f * sref[c], gl1 = 2.f * sref[c + 1];
          gam0 = __expf(gx.x);
          gam1 = __expf(gx.y);
          psi0 = __expf(gl0 - gx.x);
          psi1 = __expf(gl1 - gx.y);
          ka[b] = pack_bf16(kx.x, kx.y);  // raw k / q staged for the exact path
          qa[b] = pack_bf16(qx.x, qx.y);
          kb[b] = 0u;
        }
        qd[b] = pack_bf16(qx.x * gam0, qx.y * gam1);
        kg[b] = pack_bf16(kx.x * gam0, kx.y * gam1);
        kt[b] = pack_bf16(kx.x * psi0, kx.y * psi1);
        vv[b] = pack_bf16(vx.x, vx.y);
      }
      // non-transposed [r][c] tiles: matrix li covers columns 32cb + 8li
      const uint32_t a_rc128 = core_off(8 * warp + lr, 32 * cb + 8 * li, 128);
      if (!slow) {
        stmatrix_x4(s_base + P_KQA + a_rc128, ka[0], ka[1], ka[2], ka[3]);
        stmatrix_x4(s_base + P_KQA + core_off(64 + 8 * warp + lr, 32 * cb + 8 * li, 128), qa[0], qa[1], qa[2],
                    qa[3]);
        stmatrix_x4(s_base + P_KB + a_rc128, kb[0], kb[1], kb[2], kb[3]);
      } else {
        // plain row-major bf16 staging of k (first 16 KB) and q (next 16 KB)
        const uint32_t rowk = P_KQA + (8 * warp + lr) * 256 + (32 * cb + 8 * li) * 2;
        stmatrix_x4(s_base + rowk, ka[0], ka[1], ka[2], ka[3]);
        stmatrix_x4(s_base + rowk + 16384, qa[0], qa[1], qa[2], qa[3]);
      }
      stmatrix_x4(s_base + P_SLOT + BO_OFF + a_rc128, qd[0], qd[1], qd[2], qd[3]);
      // transposed [c][r] tiles (kdim 64): matrix li holds channels 32cb + 8li + (0..7)
      const uint32_t a_cr64 = core_off(32 * cb + 8 * li + lr, 8 * warp, 64);
      stmatrix_x4_trans(s_base + P_KGT + a_cr64, kg[0], kg[1], kg[2], kg[3]);
      stmatrix_x4_trans(s_base + P_SLOT + BS_OFF + a_cr64, kt[0], kt[1], kt[2], kt[3]);
      stmatrix_x4_trans(s_base + P_SLOT + AV_OFF + a_cr64, vv[0], vv[1], vv[2], vv[3]);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  float* Af = reinterpret_cast<float*>(smem + P_AF);
  float* Tf = reinterpret_cast<float*>(smem + P_TF);
  float* Xs = reinterpret_cast<float*>(smem + P_X);

  if (!slow) {
    // ---- A_raw / P_raw = [K o e1 ; Q o e1] (K o e2)^T on the tensor core ----
    if (tid == 0) {
      constexpr uint32_t idesc = make_idesc_bf16(128, 64);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ad = make_sdesc(s_base + P_KQA + kk * 256, 128, 2048);
        const uint64_t bd = make_sdesc(s_base + P_KB + kk * 256, 128, 2048);
        mma_bf16_ss(tmem, ad, bd, idesc, kk > 0);
      }
      mma_commit(bar_ap);
    }
    if (warp < 4) {
      mbar_wait_warp(bar_ap, 0, abort_flag);
      tc_fence_after();
      float x0[32], x1[32];
      const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16);
      tmem_ld32(ta, x0);
      tmem_ld32(ta + 32, x1);
      tmem_wait_ld();
      const int row = 32 * warp + lane;
      if (row < 64) {
        const int r = row;
        const float br = sbeta[r];
        // A overwrites the K/Q operand tiles; the MMA that read them is done
        float* arow = Af + r * AST;
#pragma unroll
        for (int s = 0; s < 32; ++s) arow[s] = s < r ? br * x0[s] : 0.f;
#pragma unroll
        for (int s = 0; s < 32; ++s) arow[32 + s] = (32 + s) < r ? br * x1[s] : 0.f;
      } else {
        const int r = row - 64;
        uint8_t* bp = slot + BP_OFF;
#pragma unroll
        for (int s8 = 0; s8 < 8; ++s8) {
          float e[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int s = 8 * s8 + u;
            const float val = s < 32 ? x0[s] : x1[s - 32];
            e[u] = s <= r ? val : 0.f;
          }
          uint4 pk;
          pk.x = pack_bf16(e[0], e[1]);
          pk.y = pack_bf16(e[2], e[3]);
          pk.z = pack_bf16(e[4], e[5]);
          pk.w = pack_bf16(e[6], e[7]);
          *reinterpret_cast<uint4*>(bp + core_off(r, 8 * s8, 64)) = pk;
        }
      }
    }
  } else {
    // ---- exact CUDA-core A and P: sum_c x_rc k_sc exp(g_rc - g_sc) -----------
    const __nv_bfloat16* ks = reinterpret_cast<const __nv_bfloat16*>(smem + P_KQA);
    const __nv_bfloat16* qs = ks + 64 * 128;
    float av[16], pv[16];
#pragma unroll 1
    for (int i = 0; i < 16; ++i) {
      const int p = tid + 256 * i;
      const int r = p >> 6, s = p & 63;
      float a = 0.f, pp = 0.f;
      if (s <= r) {
        for (int c = 0; c < 128; ++c) {
          const float e = __expf(G[r * GST + c] - G[s * GST + c]);
          const float kse = __bfloat162float(ks[s * 128 + c]) * e;
          a += __bfloat162float(ks[r * 128 + c]) * kse;
          pp += __bfloat162float(qs[r * 128 + c]) * kse;
        }
      }
      av[i] = s < r ? sbeta[r] * a : 0.f;
      pv[i] = pp;
    }
    __syncthreads();  // staged k / q are dead; A overwrites them
#pragma unroll 1
    for (int i = 0; i < 16; ++i) {
      const int p = tid + 256 * i;
      const int r = p >> 6, s = p & 63;
      Af[r * AST + s] = av[i];
      __nv_bfloat16* bp = reinterpret_cast<__nv_bfloat16*>(slot + BP_OFF + core_off(r, s, 64));
      *bp = __float2bfloat16_rn(pv[i]);
    }
  }
  __syncthreads();

  // ---- T = (I + A)^-1 by blocked forward substitution (fp32) ----------------
  if (warp < 4) {
    // diagonal 16x16 blocks: lane j < 16 solves column j of block `warp`
    const int I = warp, j = lane;
    if (j < 16) {
      float x[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < i; ++m) acc -= Af[(16 * I + i) * AST + 16 * I + m] * x[m];
        x[i] = acc;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) Tf[(16 * I + i) * AST + 16 * I + j] = x[i];
    }
  } else {
    // zero the strictly upper off-diagonal blocks of T
    for (int e = tid - 128; e < 64 * 64; e += 128) {
      const int r = e >> 6, s = e & 63;
      if ((s >> 4) > (r >> 4)) Tf[r * AST + s] = 0.f;
    }
  }
  __syncthreads();
  {
    const int i = tid >> 4, j = tid & 15;
    for (int d = 1; d < 4; ++d) {
      // X_b = sum_{K=J}^{I-1} A_IK T_KJ for blocks (I, J = I - d)
      for (int I = d, b = 0; I < 4; ++I, ++b) {
        const int J = I - d;
        float acc = 0.f;
        for (int K = J; K < I; ++K) {
#pragma unroll
          for (int m = 0; m < 16; ++m) acc += Af[(16 * I + i) * AST + 16 * K + m] * Tf[(16 * K + m) * AST + 16 * J + j];
        }
        Xs[(b * 16 + i) * 17 + j] = acc;
      }
      __syncthreads();
      // T_IJ = -T_II X_b
      for (int I = d, b = 0; I < 4; ++I, ++b) {
        const int J = I - d;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) acc += Tf[(16 * I + i) * AST + 16 * I + m] * Xs[(b * 16 + m) * 17 + j];
        Tf[(16 * I + i) * AST + 16 * J + j] = -acc;
      }
      __syncthreads();
    }
  }
  // ---- Tb = T Diag(beta) -> bf16 into the slot's U tile, columns 0..63 ------
  for (int e = tid; e < 64 * 8; e += 256) {
    const int r = e >> 3, s8 = e & 7;
    float x[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = Tf[r * AST + 8 * s8 + u] * sbeta[8 * s8 + u];
    uint4 pk;
    pk.x = pack_bf16(x[0], x[1]);
    pk.y = pack_bf16(x[2], x[3]);
    pk.z = pack_bf16(x[4], x[5]);
    pk.w = pack_bf16(x[6], x[7]);
    *reinterpret_cast<uint4*>(slot + BU_OFF + core_off(r, 8 * s8, 192)) = pk;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- W = Tb (K o Gamma) on the tensor core (M = 64, N = 128, K = 64) ------
  if (tid == 0) {
    constexpr uint32_t idesc = make_idesc_bf16(64, 128);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint64_t ad = make_sdesc(s_base + P_SLOT + BU_OFF + kk * 256, 128, 3072);
      const uint64_t bd = make_sdesc(s_base + P_KGT + kk * 256, 128, 1024);
      mma_bf16_ss(tmem + 64, ad, bd, idesc, kk > 0);
    }
    mma_commit(bar_w);
  }
  if (warp < 4) {
    mbar_wait_warp(bar_w, 0, abort_flag);
    tc_fence_after();
    // M = 64 accumulator: row 16w + i lives in TMEM lane 32w + i (i < 16)
    const uint32_t ta = tmem + (static_cast<uint32_t>(32 * warp) << 16) + 64;
    const int r = 16 * warp + lane;
#pragma unroll
    for (int cq = 0; cq < 4; ++cq) {
      float x[32];
      tmem_ld32(ta + 32 * cq, x);
      tmem_wait_ld();
      if (lane < 16) {
#pragma unroll
        for (int c8 = 0; c8 < 4; ++c8) {
          uint4 pk;
          pk.x = pack_bf16(-x[8 * c8 + 0], -x[8 * c8 + 1]);
          pk.y = pack_bf16(-x[8 * c8 + 2], -x[8 * c8 + 3]);
          pk.z = pack_bf16(-x[8 * c8 + 4], -x[8 * c8 + 5]);
          pk.w = pack_bf16(-x[8 * c8 + 6], -x[8 * c8 + 7]);
          *reinterpret_cast<uint4*>(slot + BU_OFF + core_off(r, 64 + 32 * cq + 8 * c8, 192)) = pk;
        }
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ---- publish the slot ------------------------------------------------------
  if (tid == 0) {
    uint8_t* dst = ws + (static_cast<size_t>(g) * H + h) * SLOT_BYTES;
    bulk_s2g(dst, slot, SLOT_BYTES);
    bulk_commit();
    bulk_wait_all();
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ===========================================================================
// recurrence: one CTA per (head h = blockIdx.x, sequence n = blockIdx.y)
//   warps 0-7: state / epilogue   warp 8: slot producer   warp 9: MMA issuer
// ===========================================================================
constexpr int REC_THREADS = 320;
constexpr uint32_t R_SLOT0 = 0;
constexpr uint32_t R_SLOT1 = SLOT_BYTES;
constexpr uint32_t R_TS = 2 * SLOT_BYTES;        // [128 v][128 c] bf16  S^T
constexpr uint32_t R_TU = R_TS + 32768;          // [128 v][64 r]  bf16  U^T
constexpr uint32_t R_BAR = R_TU + 16384;
constexpr uint32_t R_SMEM = R_BAR + 128;
// TMEM columns: two D1 buffers (U^T in [0,64), O^T in [64,128) of each) at
// 0 and 256, and dS^T at [128, 256).
__host__ __device__ constexpr uint32_t tm_d1(int b) { return b ? 256u : 0u; }
constexpr uint32_t TM_D2 = 128;

template <typename TIO>
__global__ void __launch_bounds__(REC_THREADS, 1)
    kda_chunk_rec_kernel(int N, int T, int H, const int32_t* __restrict__ cu, const uint8_t* __restrict__ ws,
                         const float* __restrict__ S0, TIO* __restrict__ o, float* __restrict__ S_T) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, n = blockIdx.y;

  // sequence extent and its first chunk in the flattened chunk list
  int64_t s_begin, s_end;
  int cbase = 0;
  for (int m = 0; m < n; ++m) {
    const int64_t a = cu ? cu[m] : static_cast<int64_t>(m) * T;
    const int64_t b = cu ? cu[m + 1] : a + T;
    cbase += static_cast<int>((b - a + C - 1) / C);
  }
  s_begin = cu ? cu[n] : static_cast<int64_t>(n) * T;
  s_end = cu ? cu[n + 1] : s_begin + T;
  const int nchunks = static_cast<int>((s_end - s_begin + C - 1) / C);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + R_BAR);
  uint64_t* slot_full = bars;       // [2]
  uint64_t* slot_empty = bars + 2;  // [2]
  uint64_t* d1_full = bars + 4;
  uint64_t* d2_full = bars + 5;
  uint64_t* u_ready = bars + 6;
  uint64_t* s_ready = bars + 7;
  uint64_t* d1_free = bars + 8;     // [2]
  uint64_t* fin = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 12);
  const uint32_t s_base = smem_u32(smem);

  if (tid == 0) {
    mbar_init(&slot_full[0], 1);
    mbar_init(&slot_full[1], 1);
    mbar_init(&slot_empty[0], 1 + 256);
    mbar_init(&slot_empty[1], 1 + 256);
    mbar_init(d1_full, 1);
    mbar_init(d2_full, 1);
    mbar_init(u_ready, 256);
    mbar_init(s_ready, 256);
    mbar_init(&d1_free[0], 256);
    mbar_init(&d1_free[1], 256);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const size_t slot_stride = static_cast<size_t>(H) * SLOT_BYTES;
  const uint8_t* ws_seq = ws + (static_cast<size_t>(cbase) * H + h) * SLOT_BYTES;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < nchunks; ++j) {
        const int s = j & 1;
        if (j >= 2 && !mbar_wait(&slot_empty[s], ((j - 2) >> 1) & 1, abort_flag)) break;
        issued = j + 1;
        uint8_t* dst = smem + (s ? R_SLOT1 : R_SLOT0);
        const uint8_t* src = ws_seq + static_cast<size_t>(j) * slot_stride;
        mbar_arrive_expect_tx(&slot_full[s], SLOT_BYTES);
        bulk_g2s(dst, src, 40960, &slot_full[s]);
        bulk_g2s(dst + 40960, src + 40960, SLOT_BYTES - 40960, &slot_full[s]);
      }
      // drain: copies still landing in shared memory must finish before exit
      for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&slot_full[j & 1], (j >> 1) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t id_n64 = make_idesc_bf16(128, 64);
      constexpr uint32_t id_n128 = make_idesc_bf16(128, 128);
      for (int j = 0; j < nchunks; ++j) {
        const int s = j & 1, b = j & 1;
        const uint32_t slot = s_base + (s ? R_SLOT1 : R_SLOT0);
        const uint32_t d1 = tmem + tm_d1(b);
        if (!mbar_wait(&slot_full[s], (j >> 1) & 1, abort_flag)) break;
        if (j >= 2 && !mbar_wait(&d1_free[b], ((j >> 1) - 1) & 1, abort_flag)) break;
        tc_fence_after();
        // U^T = V^T Tb^T  (K-steps over the chunk's tokens)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(d1, make_sdesc(slot + AV_OFF + kk * 256, 128, 1024),
                      make_sdesc(slot + BU_OFF + kk * 256, 128, 3072), id_n64, kk > 0);
        if (!mbar_wait(s_ready, j & 1, abort_flag)) break;
        tc_fence_after();
        // U^T += S^T (-W)^T ;  O1^T = S^T (Q o Gamma)^T
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(d1, make_sdesc(s_base + R_TS + kk * 256, 128, 2048),
                      make_sdesc(slot + BU_OFF + (4 + kk) * 256, 128, 3072), id_n64, 1);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(d1 + 64, make_sdesc(s_base + R_TS + kk * 256, 128, 2048),
                      make_sdesc(slot + BO_OFF + kk * 256, 128, 2048), id_n64, kk > 0);
        mma_commit(d1_full);
        if (!mbar_wait(u_ready, j & 1, abort_flag)) break;
        tc_fence_after();
        // dS^T = U^T (K o Psi) ;  O^T += U^T P^T
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(tmem + TM_D2, make_sdesc(s_base + R_TU + kk * 256, 128, 1024),
                      make_sdesc(slot + BS_OFF + kk * 256, 128, 1024), id_n128, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(d1 + 64, make_sdesc(s_base + R_TU + kk * 256, 128, 1024),
                      make_sdesc(slot + BP_OFF + kk * 256, 128, 1024), id_n64, 1);
        mma_commit(d2_full);
        mma_commit(&slot_empty[s]);
      }
      mma_commit(fin);
      // drain: every MMA issued above must finish before TMEM is released
      const long long t0 = clock64();
      while (!mbar_try_wait(fin, 0) && clock64() - t0 < kWaitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ state warps
    const int qd = warp & 3, hf = warp >> 2;
    const int v = 32 * qd + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * qd) << 16);
    float S[64];  // S^T[v][c], c in [64 hf, 64 hf + 64)
    const size_t sidx = (static_cast<size_t>(n) * H + h) * D * D;
    if (S0) {
#pragma unroll
      for (int i = 0; i < 64; ++i) S[i] = S0[sidx + static_cast<size_t>(64 * hf + i) * D + v];
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) S[i] = 0.f;
    }
    auto write_ST = [&]() {
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint4 pk;
        pk.x = pack_bf16(S[8 * c8 + 0], S[8 * c8 + 1]);
        pk.y = pack_bf16(S[8 * c8 + 2], S[8 * c8 + 3]);
        pk.z = pack_bf16(S[8 * c8 + 4], S[8 * c8 + 5]);
        pk.w = pack_bf16(S[8 * c8 + 6], S[8 * c8 + 7]);
        *reinterpret_cast<uint4*>(smem + R_TS + core_off(v, 64 * hf + 8 * c8, 128)) = pk;
      }
    };
    write_ST();
    fence_proxy_async_smem();
    mbar_arrive(s_ready);

    for (int j = 0; j < nchunks; ++j) {
      const int s = j & 1, b = j & 1;
      const uint8_t* slotp = smem + (s ? R_SLOT1 : R_SLOT0);
      const int64_t t0 = s_begin + static_cast<int64_t>(j) * C;
      const int64_t rem = s_end - t0;
      const int L = rem < C ? static_cast<int>(rem) : C;
      const uint32_t d1 = lane_base + tm_d1(b);

      // U^T -> bf16 operand
      if (!mbar_wait_warp(d1_full, j & 1, abort_flag)) break;
      tc_fence_after();
      {
        float x[32];
        tmem_ld32(d1 + 32 * hf, x);
        tmem_wait_ld();
#pragma unroll
        for (int r8 = 0; r8 < 4; ++r8) {
          uint4 pk;
          pk.x = pack_bf16(x[8 * r8 + 0], x[8 * r8 + 1]);
          pk.y = pack_bf16(x[8 * r8 + 2], x[8 * r8 + 3]);
          pk.z = pack_bf16(x[8 * r8 + 4], x[8 * r8 + 5]);
          pk.w = pack_bf16(x[8 * r8 + 6], x[8 * r8 + 7]);
          *reinterpret_cast<uint4*>(smem + R_TU + core_off(v, 32 * hf + 8 * r8, 64)) = pk;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(u_ready);

      // S <- gamma_C S + dS ; bf16 S^T for the next chunk
      if (!mbar_wait_warp(d2_full, j & 1, abort_flag)) break;
      tc_fence_after();
      {
        const float* gC = reinterpret_cast<const float*>(slotp + GC_OFF) + 64 * hf;
        float x[32];
        tmem_ld32(lane_base + TM_D2 + 64 * hf, x);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) S[i] = gC[i] * S[i] + x[i];
        tmem_ld32(lane_base + TM_D2 + 64 * hf + 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) S[32 + i] = gC[32 + i] * S[32 + i] + x[i];
      }
      write_ST();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(s_ready);
      mbar_arrive(&slot_empty[s]);

      // O^T -> output rows of this chunk
      {
        float x[32];
        tmem_ld32(d1 + 64 + 32 * hf, x);
        tmem_wait_ld();
        TIO* op = o + (t0 * H + h) * D + v;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int r = 32 * hf + i;
          if (r < L) st_out(op + static_cast<int64_t>(r) * H * D, x[i]);
        }
      }
      tc_fence_before();
      mbar_arrive(&d1_free[b]);
    }
    if (S_T) {
#pragma unroll
      for (int i = 0; i < 64; ++i) S_T[sidx + static_cast<size_t>(64 * hf + i) * D + v] = S[i];
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace kda
