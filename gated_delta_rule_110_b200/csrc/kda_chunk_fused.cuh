// kda_chunk_fused.cuh -- single-kernel chunkwise KDA prefill on sm_100a.
//
// One CTA per (sequence n, head h) walks the chunks of its sequence.  Inside
// the CTA three roles run concurrently, synchronised by mbarriers:
//
//   prep  (8 warps)  builds the state-independent operands of chunk j+1
//                    while the recurrence works on chunk j (a1-a4):
//                    log-decay cumsum (warp shuffles + a cross-warp prefix),
//                    the scaled operand tiles via stmatrix, A/P on tcgen05,
//                    T = (I + A)^-1 by blocked forward substitution, and
//                    W'^T on tcgen05 -- all into a double-buffered smem slot.
//   state (4 warps)  one TMEM lane per value column v.  The fp32 state S^T
//                    lives in TMEM as an MMA accumulator; per chunk the warps
//                    rescale it, write bf16 copies of S'^T, V^T and U^T back
//                    into TMEM as MMA A operands, and stream o out (a5-a7).
//   issue (2 warps)  one thread issues the recurrence MMAs, one the prep MMAs.
//
// Algebra (derivation from the recurrence S_t = (I - b k k^T) Diag(a) S + b k v^T,
// o_t = S_t^T q_t; chunk of C = 64 tokens r, g = cumsum(log a) per channel,
// per-channel reference ref = g_last / 2, sc = e^ref, e1 = e^{g - ref},
// e2 = e^{ref - g}):
//   Ka = K o e1, Qa = Q o e1, Kb = K o e2, Kt = Kb Diag(sc) = K o e^{g_last - g}
//   A  = strict_tril(Diag(b) Ka Kb^T),  P = tril(Qa Kb^T)      (one M=128 MMA)
//   T  = (I + A)^-1, Tb = T Diag(b),  W' = Tb Ka                (W'^T: M=128 MMA)
//   S' = Diag(sc) S
//   U  = Tb V - W' S'                                           (U^T = [V^T|S'^T][Tb|-W']^T)
//   O  = Qa S' + P U
//   S  <- Diag(gamma_C) S + Kt^T U                              (accumulated in TMEM)
// Chunks whose total decay exceeds the factorised range (kDecaySpan2, in log2
// units) use an exact CUDA-core A/P (2^{g_r - g_s} per term) with sc = 1.
#pragma once

#include "kda_ptx.cuh"

namespace kda {
namespace fused {

constexpr int C = 64;
constexpr int D = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kDecaySpan2 = 230.0f;  // max chunk decay in log2 units (~160 nats)

// ---- operand slot of one chunk (double-buffered) ---------------------------
constexpr uint32_t S_KA = 0;        // [64 s][128 c] K o e1      (AP A rows 0-63; W'^T A, MN-major)
constexpr uint32_t S_QA = 16384;    // [64 r][128 c] Q o e1      (AP A rows 64-127; O1 B)
constexpr uint32_t S_KT = 32768;    // [64 r][128 c] K o e^{g_last-g}  (dS B, MN-major)
constexpr uint32_t S_TB = 49152;    // [64 r][64 s]  T Diag(b)   (U B, V part; W'^T B)
constexpr uint32_t S_WT = 57344;    // [128 c][64 r] -W'^T       (U B, S part, MN-major)
constexpr uint32_t S_P = 73728;     // [64 r'][64 r] P           (O2 B)
constexpr uint32_t S_VEC = 81920;   // float sc[128], gC[128]
constexpr uint32_t SLOT = 82944;

// ---- shared memory map -----------------------------------------------------
constexpr uint32_t M_SLOT0 = 0;
constexpr uint32_t M_SLOT1 = SLOT;
constexpr uint32_t M_KB = 2 * SLOT;                 // [64 s][128 c] K o e2 (AP B)
constexpr int AST = 65;
constexpr uint32_t M_AF = M_KB + 16384;             // fp32 [64][AST] A
constexpr uint32_t M_TF = M_AF + 64 * AST * 4;      // fp32 [64][AST] T
constexpr uint32_t M_X = M_TF + 64 * AST * 4;       // fp32 [3][16][17]
constexpr uint32_t M_SCAN = M_X + 3 * 16 * 17 * 4;  // fp32 [8][128] warp totals / prefixes
constexpr uint32_t M_REF = M_SCAN + 8 * 128 * 4;    // fp32 ref2[128] (log2 units)
constexpr uint32_t M_SCF = M_REF + 128 * 4;         // fp32 2^ref2[128] (fast-path sc)
constexpr uint32_t M_BETA = M_SCF + 128 * 4;        // fp32 beta[64]
constexpr uint32_t M_FLAG = M_BETA + 64 * 4;        // int slow flag
constexpr uint32_t M_BAR = M_FLAG + 16;             // mbarriers
constexpr int NBAR = 16;
constexpr uint32_t M_TMEMSLOT = M_BAR + NBAR * 8;
constexpr uint32_t M_ABORT = M_TMEMSLOT + 4;
constexpr uint32_t SMEM_BYTES = M_ABORT + 12;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(M_BAR % 8 == 0, "mbarrier alignment");

// ---- TMEM columns ------------------------------------------------------------
constexpr uint32_t T_S = 0;      // fp32 S^T[v][c]                 128 cols
constexpr uint32_t T_SA = 128;   // bf16 pairs S'^T[v][c]            64 cols (A operand)
constexpr uint32_t T_UA = 192;   // bf16 pairs U^T[v][r]             32 cols (A operand)
constexpr uint32_t T_U = 224;    // fp32 U^T[v][r]                   64 cols
constexpr uint32_t T_O = 288;    // fp32 O^T[v][r]                   64 cols
constexpr uint32_t T_AP = 352;   // fp32 [A_raw; P_raw] (prep)       64 cols
constexpr uint32_t T_W = 416;    // fp32 W'^T[c][r] (prep)           64 cols
constexpr uint32_t T_VA = 480;   // bf16 pairs V^T[v][s]             32 cols (A operand)
constexpr uint32_t TMEM_COLS = 512;

// ---- threads -----------------------------------------------------------------
constexpr int NTHREADS = 448;  // warps 0-3 state, 4-11 prep, 12 rec issue, 13 prep issue
constexpr int PREP_THREADS = 256;

// barrier indices
enum {
  B_SLOT_FULL = 0,   // [2]  prep -> state / issue
  B_SLOT_FREE = 2,   // [2]  rec MMAs + state -> prep
  B_AP_GO = 4, B_AP_FULL, B_W_GO, B_W_FULL,
  B_S_READY, B_U_FULL, B_U_READY, B_S_FULL, B_O_FULL, B_O_FREE, B_FIN_REC, B_FIN_PREP
};

constexpr uint32_t IDESC_A_MN = 1u << 15;
constexpr uint32_t IDESC_B_MN = 1u << 16;

__device__ __forceinline__ void prep_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ bool prep_bar_or(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, 1, 256, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(p))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, "
      "%9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st32f(uint32_t taddr, const float (&f)[32]) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(f);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <typename TG>
__device__ __forceinline__ float gate_f(const TG* p);
template <>
__device__ __forceinline__ float gate_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float gate_f<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename TG>
__device__ __forceinline__ float2 gate_pair(const TG* p);
template <>
__device__ __forceinline__ float2 gate_pair<float>(const float* p) { return make_float2(p[0], p[1]); }
template <>
__device__ __forceinline__ float2 gate_pair<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}

__device__ __forceinline__ float2 bf2(uint32_t u) {
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(b);
}

// Sequence extent of CTA's sequence n.
__device__ __forceinline__ void seq_extent(int n, int T, const int32_t* cu, int64_t* b, int64_t* e) {
  *b = cu ? cu[n] : static_cast<int64_t>(n) * T;
  *e = cu ? cu[n + 1] : *b + T;
}

// ============================================================================
// prep role: 256 threads (warps 4-11).  pw = warp - 4 owns rows 8pw..8pw+7.
// ============================================================================
template <typename TG>
__device__ __forceinline__ void prep_role(uint8_t* smem, uint32_t s_base, uint32_t tmem, int nc, int64_t s_begin,
                                          int64_t s_end, int h, int H, const __nv_bfloat16* __restrict__ q,
                                          const __nv_bfloat16* __restrict__ k, const TG* __restrict__ la,
                                          const TG* __restrict__ beta, uint64_t* bars, volatile int* abort_flag) {
  const int ptid = threadIdx.x - 128;  // 0..255
  const int pw = ptid >> 5, lane = ptid & 31;
  const int rr = lane >> 2, cc = (lane & 3) * 2;
  const int r = 8 * pw + rr;
  const uint32_t li = lane >> 3, lr = lane & 7;
  float* scan = reinterpret_cast<float*>(smem + M_SCAN);
  float* ref2s = reinterpret_cast<float*>(smem + M_REF);
  float* sbeta = reinterpret_cast<float*>(smem + M_BETA);
  volatile int* sflag = reinterpret_cast<volatile int*>(smem + M_FLAG);
  float* Af = reinterpret_cast<float*>(smem + M_AF);
  float* Tf = reinterpret_cast<float*>(smem + M_TF);
  float* Xs = reinterpret_cast<float*>(smem + M_X);

  for (int j = 0; j < nc; ++j) {
    const int s = j & 1;
    const uint32_t slot_off = s ? M_SLOT1 : M_SLOT0;
    uint8_t* slot = smem + slot_off;
    const uint32_t slot_a = s_base + slot_off;
    const int64_t t0 = s_begin + static_cast<int64_t>(j) * C;
    const int64_t rem = s_end - t0;
    const int L = rem < C ? static_cast<int>(rem) : C;
    const bool live = r < L;
    const int64_t grow = (t0 + r) * H + h;

    // ---- global loads: log-decay, k, q in stmatrix fragment layout --------
    float lg[32];
    uint32_t kr[16], qr[16];
#pragma unroll
    for (int cb = 0; cb < 4; ++cb)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int c = 32 * cb + 8 * b + cc;
        const int i = 4 * cb + b;
        if (live) {
          const float2 l2 = gate_pair(la + grow * D + c);
          lg[2 * i] = l2.x * kLog2e;
          lg[2 * i + 1] = l2.y * kLog2e;
          kr[i] = *reinterpret_cast<const uint32_t*>(k + grow * D + c);
          qr[i] = *reinterpret_cast<const uint32_t*>(q + grow * D + c);
        } else {
          lg[2 * i] = lg[2 * i + 1] = 0.f;
          kr[i] = qr[i] = 0u;
        }
      }
    if ((lane & 3) == 0) sbeta[r] = live ? gate_f(beta + grow) : 0.f;

    // the slot must be released by the recurrence two chunks back
    if (j >= 2) mbar_wait_warp(&bars[B_SLOT_FREE + s], ((j - 2) >> 1) & 1, abort_flag);

    // ---- inclusive cumsum over the chunk, per channel (log2 units) ---------
#pragma unroll
    for (int i = 0; i < 32; ++i) {
#pragma unroll
      for (int d = 4; d < 32; d <<= 1) {
        const float up = __shfl_up_sync(0xffffffffu, lg[i], d);
        if (lane >= d) lg[i] += up;
      }
    }
    if (rr == 7) {
#pragma unroll
      for (int cb = 0; cb < 4; ++cb)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int c = 32 * cb + 8 * b + cc;
          const int i = 4 * cb + b;
          scan[pw * 128 + c] = lg[2 * i];
          scan[pw * 128 + c + 1] = lg[2 * i + 1];
        }
    }
    prep_bar();
    bool slow_c = false;
    if (ptid < 128) {
      float run = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float x = scan[w * 128 + ptid];
        scan[w * 128 + ptid] = run;
        run += x;
      }
      ref2s[ptid] = 0.5f * run;
      reinterpret_cast<float*>(smem + M_SCF)[ptid] = ex2(0.5f * run);
      slow_c = -run > kDecaySpan2;
      reinterpret_cast<float*>(slot + S_VEC)[128 + ptid] = ex2(run);  // gamma_C
    }
    const bool slow = prep_bar_or(slow_c);
    const float* scf = reinterpret_cast<const float*>(smem + M_SCF);
    if (ptid < 128) reinterpret_cast<float*>(slot + S_VEC)[ptid] = slow ? 1.f : scf[ptid];  // sc
    // add the exclusive prefix of the earlier row blocks
#pragma unroll
    for (int cb = 0; cb < 4; ++cb)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int c = 32 * cb + 8 * b + cc;
        const int i = 4 * cb + b;
        const float2 pf = *reinterpret_cast<const float2*>(scan + pw * 128 + c);
        lg[2 * i] += pf.x;
        lg[2 * i + 1] += pf.y;
      }

    if (!slow) {
      // ---- operand tiles: Ka, Qa (slot), Kb (scratch), Kt (slot) -----------
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t ka[4], qa[4], kb[4], kt[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int i = 4 * cb + b;
          const int c = 32 * cb + 8 * b + cc;
          const float2 kx = bf2(kr[i]), qx = bf2(qr[i]);
          const float2 rf = *reinterpret_cast<const float2*>(ref2s + c);
          const float2 sf = *reinterpret_cast<const float2*>(scf + c);
          const float e10 = ex2(lg[2 * i] - rf.x), e11 = ex2(lg[2 * i + 1] - rf.y);
          const float e20 = ex2(rf.x - lg[2 * i]), e21 = ex2(rf.y - lg[2 * i + 1]);
          const float s0 = sf.x, s1 = sf.y;
          ka[b] = pack_bf16(kx.x * e10, kx.y * e11);
          qa[b] = pack_bf16(qx.x * e10, qx.y * e11);
          kb[b] = pack_bf16(kx.x * e20, kx.y * e21);
          kt[b] = pack_bf16(kx.x * e20 * s0, kx.y * e21 * s1);
        }
        const uint32_t a_rc = core_off(8 * pw + lr, 32 * cb + 8 * li, 128);
        stmatrix_x4(slot_a + S_KA + a_rc, ka[0], ka[1], ka[2], ka[3]);
        stmatrix_x4(slot_a + S_QA + a_rc, qa[0], qa[1], qa[2], qa[3]);
        stmatrix_x4(s_base + M_KB + a_rc, kb[0], kb[1], kb[2], kb[3]);
        stmatrix_x4(slot_a + S_KT + a_rc, kt[0], kt[1], kt[2], kt[3]);
      }
      fence_proxy_async_smem();
      prep_bar();
      if (ptid == 0) {
        *sflag = 0;
        mbar_arrive(&bars[B_AP_GO]);
      }
      // ---- A / P epilogue ----------------------------------------------------
      mbar_wait_warp(&bars[B_AP_FULL], j & 1, abort_flag);
      tc_fence_after();
      {
        const int qd = pw & 3, hf = pw >> 2;
        const int row = 32 * qd + lane;
        float x[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * qd) << 16) + T_AP + 32 * hf, x);
        tmem_wait_ld();
        if (row < 64) {
          const float br = sbeta[row];
          float* arow = Af + row * AST + 32 * hf;
#pragma unroll
          for (int u = 0; u < 32; ++u) arow[u] = (32 * hf + u) < row ? br * x[u] : 0.f;
        } else {
          const int rp = row - 64;
#pragma unroll
          for (int u8 = 0; u8 < 4; ++u8) {
            float e[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) e[u] = (32 * hf + 8 * u8 + u) <= rp ? x[8 * u8 + u] : 0.f;
            uint4 pk;
            pk.x = pack_bf16(e[0], e[1]);
            pk.y = pack_bf16(e[2], e[3]);
            pk.z = pack_bf16(e[4], e[5]);
            pk.w = pack_bf16(e[6], e[7]);
            *reinterpret_cast<uint4*>(slot + S_P + core_off(rp, 32 * hf + 8 * u8, 64)) = pk;
          }
        }
      }
      tc_fence_before();
      prep_bar();
    } else {
      // ---- exact path: stage g (fp32, over the Ka/Qa tiles), k, q ------------
      float* G = reinterpret_cast<float*>(slot + S_KA);
      __nv_bfloat16* ks = reinterpret_cast<__nv_bfloat16*>(smem + M_KB);
      __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem + M_TF);
#pragma unroll
      for (int cb = 0; cb < 4; ++cb)
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int c = 32 * cb + 8 * b + cc;
          const int i = 4 * cb + b;
          *reinterpret_cast<float2*>(G + r * 128 + c) = make_float2(lg[2 * i], lg[2 * i + 1]);
          *reinterpret_cast<uint32_t*>(ks + r * 128 + c) = kr[i];
          *reinterpret_cast<uint32_t*>(qs + r * 128 + c) = qr[i];
        }
      prep_bar();
      float av[16], pv[16];
#pragma unroll 1
      for (int it = 0; it < 16; ++it) {
        const int p = ptid + 256 * it;
        const int ar = p >> 6, as = p & 63;
        float a = 0.f, pp = 0.f;
        if (as <= ar) {
          for (int c = 0; c < 128; ++c) {
            const float e = ex2(G[ar * 128 + c] - G[as * 128 + c]);
            const float kse = __bfloat162float(ks[as * 128 + c]) * e;
            a += __bfloat162float(ks[ar * 128 + c]) * kse;
            pp += __bfloat162float(qs[ar * 128 + c]) * kse;
          }
        }
        av[it] = as < ar ? sbeta[ar] * a : 0.f;
        pv[it] = pp;
      }
      prep_bar();  // staged g / k / q are dead from here on
#pragma unroll 1
      for (int it = 0; it < 16; ++it) {
        const int p = ptid + 256 * it;
        const int ar = p >> 6, as = p & 63;
        Af[ar * AST + as] = av[it];
        *reinterpret_cast<__nv_bfloat16*>(slot + S_P + core_off(ar, as, 64)) = __float2bfloat16_rn(pv[it]);
      }
      // operand tiles with sc = 1: Ka = K o Gamma, Qa = Q o Gamma, Kt = K o Psi
      const float* gl = reinterpret_cast<const float*>(smem + M_REF);  // ref2 = g_last / 2
#pragma unroll
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t ka[4], qa[4], kt[4];
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const int c = 32 * cb + 8 * b + cc;
          const int i = 4 * cb + b;
          const float2 kx = bf2(kr[i]), qx = bf2(qr[i]);
          const float g0 = ex2(lg[2 * i]), g1 = ex2(lg[2 * i + 1]);
          const float p0 = ex2(2.f * gl[c] - lg[2 * i]), p1 = ex2(2.f * gl[c + 1] - lg[2 * i + 1]);
          ka[b] = pack_bf16(kx.x * g0, kx.y * g1);
          qa[b] = pack_bf16(qx.x * g0, qx.y * g1);
          kt[b] = pack_bf16(kx.x * p0, kx.y * p1);
        }
        const uint32_t a_rc = core_off(8 * pw + lr, 32 * cb + 8 * li, 128);
        stmatrix_x4(slot_a + S_KA + a_rc, ka[0], ka[1], ka[2], ka[3]);
        stmatrix_x4(slot_a + S_QA + a_rc, qa[0], qa[1], qa[2], qa[3]);
        stmatrix_x4(slot_a + S_KT + a_rc, kt[0], kt[1], kt[2], kt[3]);
      }
      fence_proxy_async_smem();
      prep_bar();
      if (ptid == 0) {
        *sflag = 1;  // tell the prep issuer there is no A/P product this chunk
        mbar_arrive(&bars[B_AP_GO]);
      }
      mbar_wait_warp(&bars[B_AP_FULL], j & 1, abort_flag);
      prep_bar();
    }

    // ---- T = (I + A)^-1: diagonal 16x16 blocks, then three block levels -----
    if (pw < 4) {
      const int I = pw, jc = lane;
      if (jc < 16) {
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float acc = (i == jc) ? 1.f : 0.f;
#pragma unroll
          for (int m = 0; m < i; ++m) acc -= Af[(16 * I + i) * AST + 16 * I + m] * x[m];
          x[i] = acc;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Tf[(16 * I + i) * AST + 16 * I + jc] = x[i];
      }
    } else {
      for (int e = ptid - 128; e < 64 * 64; e += 128) {
        const int ar = e >> 6, as = e & 63;
        if ((as >> 4) > (ar >> 4)) Tf[ar * AST + as] = 0.f;
      }
    }
    prep_bar();
    {
      const int i = ptid >> 4, jj = ptid & 15;
      for (int d = 1; d < 4; ++d) {
        for (int I = d, bb = 0; I < 4; ++I, ++bb) {
          const int J = I - d;
          float acc = 0.f;
          for (int K = J; K < I; ++K) {
#pragma unroll
            for (int m = 0; m < 16; ++m)
              acc += Af[(16 * I + i) * AST + 16 * K + m] * Tf[(16 * K + m) * AST + 16 * J + jj];
          }
          Xs[(bb * 16 + i) * 17 + jj] = acc;
        }
        prep_bar();
        for (int I = d, bb = 0; I < 4; ++I, ++bb) {
          const int J = I - d;
          float acc = 0.f;
#pragma unroll
          for (int m = 0; m < 16; ++m) acc += Tf[(16 * I + i) * AST + 16 * I + m] * Xs[(bb * 16 + m) * 17 + jj];
          Tf[(16 * I + i) * AST + 16 * J + jj] = -acc;
        }
        prep_bar();
      }
    }
    // ---- Tb = T Diag(b) -> bf16 [r][s] ------------------------------------------
    for (int e = ptid; e < 64 * 8; e += 256) {
      const int ar = e >> 3, s8 = e & 7;
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = Tf[ar * AST + 8 * s8 + u] * sbeta[8 * s8 + u];
      uint4 pk;
      pk.x = pack_bf16(x[0], x[1]);
      pk.y = pack_bf16(x[2], x[3]);
      pk.z = pack_bf16(x[4], x[5]);
      pk.w = pack_bf16(x[6], x[7]);
      *reinterpret_cast<uint4*>(slot + S_TB + core_off(ar, 8 * s8, 64)) = pk;
    }
    fence_proxy_async_smem();
    prep_bar();
    if (ptid == 0) mbar_arrive(&bars[B_W_GO]);

    // ---- W'^T epilogue: -W'^T[c][r] -> bf16 [c][r] --------------------------------
    mbar_wait_warp(&bars[B_W_FULL], j & 1, abort_flag);
    tc_fence_after();
    {
      const int qd = pw & 3, hf = pw >> 2;
      const int c = 32 * qd + lane;
      float x[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * qd) << 16) + T_W + 32 * hf, x);
      tmem_wait_ld();
#pragma unroll
      for (int u8 = 0; u8 < 4; ++u8) {
        uint4 pk;
        pk.x = pack_bf16(-x[8 * u8 + 0], -x[8 * u8 + 1]);
        pk.y = pack_bf16(-x[8 * u8 + 2], -x[8 * u8 + 3]);
        pk.z = pack_bf16(-x[8 * u8 + 4], -x[8 * u8 + 5]);
        pk.w = pack_bf16(-x[8 * u8 + 6], -x[8 * u8 + 7]);
        *reinterpret_cast<uint4*>(slot + S_WT + core_off(c, 32 * hf + 8 * u8, 64)) = pk;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    prep_bar();
    if (ptid == 0) mbar_arrive(&bars[B_SLOT_FULL + s]);
  }
}

// ============================================================================
// state role: 128 threads (warps 0-3), thread v <-> TMEM lane v
// ============================================================================
template <typename TIO>
__device__ __forceinline__ void state_role(uint8_t* smem, uint32_t tmem, int nc, int64_t s_begin, int64_t s_end,
                                           int n, int h, int H, const TIO* __restrict__ v, const float* __restrict__ S0,
                                           TIO* __restrict__ o, float* __restrict__ S_T, uint64_t* bars,
                                           volatile int* abort_flag) {
  const int vv = threadIdx.x;  // 0..127
  const int warp = vv >> 5;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * warp) << 16);
  const size_t sidx = (static_cast<size_t>(n) * H + h) * D * D;

  // S0 -> TMEM S^T[v][c]
#pragma unroll 1
  for (int cb = 0; cb < 4; ++cb) {
    float x[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = S0 ? S0[sidx + static_cast<size_t>(32 * cb + i) * D + vv] : 0.f;
    tmem_st32f(lane_base + T_S + 32 * cb, x);
  }
  tmem_wait_st();

  // V prefetch: column vv of the chunk's 64 value rows, packed in pairs along the tokens
  uint32_t vpre[32];
  auto load_v = [&](int j) {
    const int64_t t0 = s_begin + static_cast<int64_t>(j) * C;
    const int64_t rem = s_end - t0;
    const int L = rem < C ? static_cast<int>(rem) : C;
    const unsigned short* vp = reinterpret_cast<const unsigned short*>(v) + (t0 * H + h) * D + vv;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const uint32_t lo = (2 * i < L) ? vp[static_cast<int64_t>(2 * i) * H * D] : 0u;
      const uint32_t hi = (2 * i + 1 < L) ? vp[static_cast<int64_t>(2 * i + 1) * H * D] : 0u;
      vpre[i] = lo | (hi << 16);
    }
  };
  if (nc > 0) load_v(0);

  auto read_o = [&](int j) {
    mbar_wait_warp(&bars[B_O_FULL], j & 1, abort_flag);
    tc_fence_after();
    const int64_t t0 = s_begin + static_cast<int64_t>(j) * C;
    const int64_t rem = s_end - t0;
    const int L = rem < C ? static_cast<int>(rem) : C;
    TIO* op = o + (t0 * H + h) * D + vv;
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      float x[32];
      tmem_ld32(lane_base + T_O + 32 * half, x);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = 32 * half + i;
        if (r < L) {
          if constexpr (sizeof(TIO) == 2)
            op[static_cast<int64_t>(r) * H * D] = __float2bfloat16_rn(x[i]);
          else
            op[static_cast<int64_t>(r) * H * D] = x[i];
        }
      }
    }
    tc_fence_before();
    mbar_arrive(&bars[B_O_FREE]);
    mbar_arrive(&bars[B_SLOT_FREE + (j & 1)]);
  };

  for (int j = 0; j < nc; ++j) {
    const int s = j & 1;
    const float* vec = reinterpret_cast<const float*>(smem + (s ? M_SLOT1 : M_SLOT0) + S_VEC);
    if (!mbar_wait_warp(&bars[B_SLOT_FULL + s], (j >> 1) & 1, abort_flag)) break;
    tc_fence_after();
    // S'^T = bf16(sc S^T) -> A operand;  S^T <- gamma_C S^T;  V^T -> A operand
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
      float x[32];
      tmem_ld32(lane_base + T_S + 32 * cb, x);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        pk[i] = pack_bf16(x[2 * i] * vec[32 * cb + 2 * i], x[2 * i + 1] * vec[32 * cb + 2 * i + 1]);
      tmem_st16(lane_base + T_SA + 16 * cb, pk);
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] *= vec[128 + 32 * cb + i];
      tmem_st32f(lane_base + T_S + 32 * cb, x);
    }
    {
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[i] = vpre[i];
      tmem_st16(lane_base + T_VA, pk);
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[i] = vpre[16 + i];
      tmem_st16(lane_base + T_VA + 16, pk);
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bars[B_S_READY]);

    if (j >= 1) read_o(j - 1);
    if (j + 1 < nc) load_v(j + 1);

    // U^T -> bf16 A operand (its previous readers, the last chunk's dS / O2
    // MMAs, were issued before the U^T MMAs this wait covers)
    if (!mbar_wait_warp(&bars[B_U_FULL], j & 1, abort_flag)) break;
    tc_fence_after();
    {
      float x[32];
      uint32_t pk[16];
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(lane_base + T_U + 32 * half, x);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(x[2 * i], x[2 * i + 1]);
        tmem_st16(lane_base + T_UA + 16 * half, pk);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    mbar_arrive(&bars[B_U_READY]);

    if (!mbar_wait_warp(&bars[B_S_FULL], j & 1, abort_flag)) break;
  }
  if (nc > 0 && !*abort_flag) read_o(nc - 1);

  // final state
  tc_fence_after();
  if (S_T) {
#pragma unroll 1
    for (int cb = 0; cb < 4; ++cb) {
      float x[32];
      tmem_ld32(lane_base + T_S + 32 * cb, x);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) S_T[sidx + static_cast<size_t>(32 * cb + i) * D + vv] = x[i];
    }
  }
}

// ============================================================================
// issue roles
// ============================================================================
__device__ __forceinline__ void rec_issue(uint32_t s_base, uint32_t tmem, int nc, uint64_t* bars,
                                          volatile int* abort_flag) {
  constexpr uint32_t id_u = make_idesc_bf16(128, 64);
  constexpr uint32_t id_u_bmn = make_idesc_bf16(128, 64) | IDESC_B_MN;
  constexpr uint32_t id_ds = make_idesc_bf16(128, 128) | IDESC_B_MN;
  for (int j = 0; j < nc; ++j) {
    const int s = j & 1;
    const uint32_t slot = s_base + (s ? M_SLOT1 : M_SLOT0);
    if (!mbar_wait(&bars[B_SLOT_FULL + s], (j >> 1) & 1, abort_flag)) break;
    if (!mbar_wait(&bars[B_S_READY], j & 1, abort_flag)) break;
    tc_fence_after();
    // U^T = V^T Tb^T (4 K-steps over tokens) - S'^T W'^T (8 K-steps over channels)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ts(tmem + T_U, tmem + T_VA + 8 * kk, make_sdesc(slot + S_TB + kk * 256, 128, 1024), id_u, kk > 0);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_ts(tmem + T_U, tmem + T_SA + 8 * kk, make_sdesc(slot + S_WT + kk * 2048, 1024, 128), id_u_bmn, 1);
    mma_commit(&bars[B_U_FULL]);
    // O1^T = S'^T Qa^T (needs the previous chunk's O read out)
    if (j >= 1 && !mbar_wait(&bars[B_O_FREE], (j - 1) & 1, abort_flag)) break;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_ts(tmem + T_O, tmem + T_SA + 8 * kk, make_sdesc(slot + S_QA + kk * 256, 128, 2048), id_u, kk > 0);
    // dS^T = U^T Kt accumulated onto gamma_C S^T ; O^T += U^T P^T
    if (!mbar_wait(&bars[B_U_READY], j & 1, abort_flag)) break;
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ts(tmem + T_S, tmem + T_UA + 8 * kk, make_sdesc(slot + S_KT + kk * 4096, 2048, 128), id_ds, 1);
    mma_commit(&bars[B_S_FULL]);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ts(tmem + T_O, tmem + T_UA + 8 * kk, make_sdesc(slot + S_P + kk * 256, 128, 1024), id_u, 1);
    mma_commit(&bars[B_O_FULL]);
    mma_commit(&bars[B_SLOT_FREE + s]);
  }
  mma_commit(&bars[B_FIN_REC]);
  const long long t0 = clock64();
  while (!mbar_try_wait(&bars[B_FIN_REC], 0) && clock64() - t0 < kWaitCycles) {
  }
}

__device__ __forceinline__ void prep_issue(uint8_t* smem, uint32_t s_base, uint32_t tmem, int nc, uint64_t* bars,
                                           volatile int* abort_flag) {
  constexpr uint32_t id_ap = make_idesc_bf16(128, 64);
  constexpr uint32_t id_w = make_idesc_bf16(128, 64) | IDESC_A_MN;
  volatile int* sflag = reinterpret_cast<volatile int*>(smem + M_FLAG);
  for (int j = 0; j < nc; ++j) {
    const int s = j & 1;
    const uint32_t slot = s_base + (s ? M_SLOT1 : M_SLOT0);
    if (!mbar_wait(&bars[B_AP_GO], j & 1, abort_flag)) break;
    tc_fence_after();
    if (*sflag == 0) {
      // [A_raw; P_raw] = [Ka; Qa] Kb^T   (M = 128, N = 64, K = 128)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tmem + T_AP, make_sdesc(slot + S_KA + kk * 256, 128, 2048),
                    make_sdesc(s_base + M_KB + kk * 256, 128, 2048), id_ap, kk > 0);
    }
    mma_commit(&bars[B_AP_FULL]);
    if (!mbar_wait(&bars[B_W_GO], j & 1, abort_flag)) break;
    tc_fence_after();
    // W'^T[c][r] = sum_s Ka[s][c] Tb[r][s]   (A = Ka MN-major, M = 128, N = 64, K = 64)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16_ss(tmem + T_W, make_sdesc(slot + S_KA + kk * 4096, 2048, 128),
                  make_sdesc(slot + S_TB + kk * 256, 128, 1024), id_w, kk > 0);
    mma_commit(&bars[B_W_FULL]);
  }
  mma_commit(&bars[B_FIN_PREP]);
  const long long t0 = clock64();
  while (!mbar_try_wait(&bars[B_FIN_PREP], 0) && clock64() - t0 < kWaitCycles) {
  }
}

// ============================================================================
// the kernel: grid (H, N), one CTA per (head, sequence)
// ============================================================================
template <typename TG>
__global__ void __launch_bounds__(NTHREADS, 1)
    kda_chunk_fused_kernel(int T, int H, const int32_t* __restrict__ cu, const __nv_bfloat16* __restrict__ q,
                           const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                           const TG* __restrict__ la, const TG* __restrict__ beta, const float* __restrict__ S0,
                           __nv_bfloat16* __restrict__ o, float* __restrict__ S_T) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, n = blockIdx.y;
  int64_t s_begin, s_end;
  seq_extent(n, T, cu, &s_begin, &s_end);
  const int nc = static_cast<int>((s_end - s_begin + C - 1) / C);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + M_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + M_TMEMSLOT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + M_ABORT);
  const uint32_t s_base = smem_u32(smem);

  if (threadIdx.x == 0) {
    mbar_init(&bars[B_SLOT_FULL + 0], 1);
    mbar_init(&bars[B_SLOT_FULL + 1], 1);
    mbar_init(&bars[B_SLOT_FREE + 0], 1 + 128);
    mbar_init(&bars[B_SLOT_FREE + 1], 1 + 128);
    mbar_init(&bars[B_AP_GO], 1);
    mbar_init(&bars[B_AP_FULL], 1);
    mbar_init(&bars[B_W_GO], 1);
    mbar_init(&bars[B_W_FULL], 1);
    mbar_init(&bars[B_S_READY], 128);
    mbar_init(&bars[B_U_FULL], 1);
    mbar_init(&bars[B_U_READY], 128);
    mbar_init(&bars[B_S_FULL], 1);
    mbar_init(&bars[B_O_FULL], 1);
    mbar_init(&bars[B_O_FREE], 128);
    mbar_init(&bars[B_FIN_REC], 1);
    mbar_init(&bars[B_FIN_PREP], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    state_role<__nv_bfloat16>(smem, tmem, nc, s_begin, s_end, n, h, H, v, S0, o, S_T, bars, abort_flag);
  } else if (warp < 12) {
    prep_role<TG>(smem, s_base, tmem, nc, s_begin, s_end, h, H, q, k, la, beta, bars, abort_flag);
  } else if (warp == 12) {
    if (lane == 0) rec_issue(s_base, tmem, nc, bars, abort_flag);
  } else {
    if (lane == 0) prep_issue(smem, s_base, tmem, nc, bars, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fused
}  // namespace kda
