// kda_prefill.cuh -- chunkwise-parallel KDA prefill on sm_100a as one
// persistent, cooperatively launched kernel with two kinds of CTA.
//
// The chunk form ("Kimi Linear" summary page, section "Algoritmo paralelo por
// chunks"): fixed chunks of C = 64 tokens, the final state of a chunk seeds the
// next, the chunk's rank-1 updates are folded into a WY / UT representation
// built with a lower-triangular inverse, and the output is an inter-chunk
// (state) term plus an intra-chunk term.  The algebra, derived here from the
// recurrence S_t = (I - b k k^T) Diag(a) S + b k v^T, o_t = S_t^T q_t, for a
// chunk with rows r, g = per-channel cumulative log decay, a per-channel
// reference ref = g_last / 2, sc = e^ref:
//   Ka = K o e^{g - ref}   Qa = Q o e^{g - ref}   Kb = K o e^{ref - g}
//   Kt = Kb Diag(sc) = K o e^{g_last - g}        gC = e^{g_last}
//   A  = strict_tril(Diag(b) Ka Kb^T)           P = tril(Qa Kb^T)
//   T  = (I + A)^-1,  Tb = T Diag(b),  W' = Tb Ka
//   S' = Diag(sc) S        (S = state at the chunk start)
//   U  = Tb V - W' S'      O = Qa S' + P U      S <- Diag(gC) S + Kt^T U
// Everything above the line "S' = ..." is independent of the state, so it is
// computed fully in parallel; only the last line is a chain over chunks.
// Chunks whose total decay exceeds the factorised range (kSpan2, log2 units,
// about 160 nats) take an exact CUDA-core A / P with sc = 1.
//
// CTA roles (grid = one CTA per SM, 384 threads, launched cooperatively so
// every CTA is resident at once):
//   * state CTAs (blockIdx < R) each own a stream of (sequence, head) chains
//     and walk their chunks in order: the fp32 state S^T lives in registers of
//     8 warps; bf16 copies of S'^T and U^T go to shared memory as MMA A
//     operands; tcgen05 computes U^T, O^T and dS^T into TMEM.
//   * transform CTAs (the rest) build the state-independent operands of one
//     chunk at a time (two independent groups per CTA): cumulative log decay
//     (a tensor-core product with a lower-triangular ones matrix), the scaled
//     tiles, A / P on tcgen05, T by blocked forward substitution on CUDA cores,
//     W'^T on tcgen05, and write them to a ring slot in global memory.
// The ring (nring <= 16 slots per state CTA, ~65 KB each) is small enough to stay in
// L2.  A transform CTA claims work items from a global counter in stream
// order; it writes a slot once the state CTA has copied the slot's previous
// contents (the `consumed` counter) and publishes it with a release store of
// the position (`ready`).  The state CTA polls `ready` with acquire loads and
// bulk-copies the slot into shared memory.  Items are claimed in increasing
// stream position, so the smallest unfinished item can always proceed: with
// every CTA resident the protocol cannot deadlock.  All waits are bounded; a
// wait that runs out records KDA_ERR_TIMEOUT and raises a global abort flag
// that every CTA polls.
#pragma once

#include "kda_epilogue.cuh"
#include "kda_ptx.cuh"
#include "kda_state_io.cuh"

namespace kda {
namespace pipe {

#ifdef KDA_TEST_HOOKS
// Test-only build: when set, state CTA 0 never signals that its first U^T is
// complete, so the state warps' bounded wait runs out (the failure-detection
// test); every other wait then ends through the abort flag or its own limit.
__device__ int g_test_skip_commit = 0;
#endif

constexpr int C = 64;
constexpr int D = 128;
constexpr int NTHREADS = 384;
constexpr int MAX_RING = 16;  // ring slots per state CTA (the host picks 2..16)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSpan2 = 230.0f;  // largest chunk decay of the factorised path, log2 units

// ---- ring slot: operands of one chunk as the state CTA's MMAs read them ----
// Part A (Tb, -W'^T, the per-channel scales) feeds U and is released once U
// is formed; part B (Qa, Kt, P) feeds the state update and the output.  The
// state CTA copies and releases the two parts separately.
constexpr uint32_t R_TB = 0;       // A: Tb [r][s] bf16, K-major                     8 KB
constexpr uint32_t R_WT = 8192;    // A: -W'^T [c][r] bf16, M/N-major B              16 KB
constexpr uint32_t R_VEC = 24576;  // A: sc[128], gC[128] fp32                        1 KB
constexpr uint32_t R_QA = 25600;   // B: Qa [r][c] bf16, two 64-channel atoms        16 KB
constexpr uint32_t R_KT = 41984;   // B: Kt [r][c] bf16, two 64-channel atoms        16 KB
constexpr uint32_t R_PP = 58368;   // B: P [r'][r] bf16, K-major                      8 KB
constexpr uint32_t SLOT = 66560;
constexpr uint32_t SLOT_A = R_QA;         // bytes of part A
constexpr uint32_t SLOT_B = SLOT - R_QA;  // bytes of part B
static_assert(R_QA % 1024 == 0 && R_KT % 1024 == 0 && R_PP % 1024 == 0 && SLOT % 1024 == 0, "tile alignment");

// ---- global flags (32-bit words) ---------------------------------------------
constexpr uint32_t F_COUNTER = 0;     // next work item
constexpr uint32_t F_ABORT = 32;      // any CTA gave up
constexpr uint32_t F_REC0 = 64;       // per state CTA: ready[nring] at +0, consumed at +32
constexpr uint32_t F_REC_STRIDE = 64;
constexpr uint32_t F_CONSUMED = 32;
__host__ __device__ constexpr size_t flag_words(int R) { return F_REC0 + static_cast<size_t>(R) * F_REC_STRIDE; }

// ---- state CTA shared memory --------------------------------------------------
constexpr uint32_t ST_A = 0;                      // 2 x part A (position parity)
constexpr uint32_t ST_V = ST_A + 2 * SLOT_A;      // 2 x V tile [r][v] (two 64-value atoms)
constexpr uint32_t ST_B = ST_V + 2 * 16384;       // 2 x part B
constexpr uint32_t ST_S = ST_B + 2 * SLOT_B;       // S'^T [v][c] bf16, two 64-channel atoms
constexpr uint32_t ST_U = ST_S + 32768;           // U^T [v][r] bf16
constexpr uint32_t ST_OX = ST_U + 16384;          // O staging of the two output warps, 2 x [32 rows][128 v] bf16
constexpr uint32_t ST_BAR = ST_OX + 16384;
constexpr uint32_t ST_W = ST_BAR + 256;           // output epilogue: norm weight fp32[128]
constexpr uint32_t ST_BYTES = ST_W + 512;
static_assert(ST_BYTES <= 227u * 1024u, "state CTA shared memory");
// TMEM columns
constexpr uint32_t TS_U = 0;     // U^T fp32                       64
constexpr uint32_t TS_DS = 128;  // dS^T fp32                     128
constexpr uint32_t TS_O = 256;   // 2 x O [r][v] fp32, row r in lane 64 + r   2 x 128

// ---- transform CTA shared memory ------------------------------------------------
template <typename TG>
struct TfLayout {
  static constexpr int NGROUP = sizeof(TG) == 2 ? 2 : 1;
  static constexpr uint32_t RL_BYTES = sizeof(TG) == 2 ? 16384 : 32768;
  static constexpr uint32_t L = 0;                       // [128][64] bf16 lower-triangular ones (twice)
  static constexpr uint32_t G_RQ = 0;                    // raw q [r][c], two atoms
  static constexpr uint32_t G_RK = 16384;                // raw k
  static constexpr uint32_t G_RL = 32768;                // raw log-decay (bf16: 2 atoms, fp32: 4 atoms)
  static constexpr uint32_t G_KQ = G_RL + RL_BYTES;      // [Ka; Qa] 2 K-atoms of [128][64]; T (fp32) later
  static constexpr uint32_t G_KB = G_KQ + 32768;         // Kb 2 atoms of [64][64]; A (fp32) later
  static constexpr uint32_t G_TB = G_KB + 16384;         // Tb [r][s]; inverse scratch before that
  static constexpr uint32_t GROUP = G_TB + 8192;
  static constexpr uint32_t GBASE = 16384;
  static constexpr uint32_t MISC = GBASE + NGROUP * GROUP;
  // per-group misc block
  static constexpr uint32_t M_BETA = 0;     // fp32[64]
  static constexpr uint32_t M_GL = 256;     // fp32[128]  g_last (log2 units)
  static constexpr uint32_t M_SC = 768;     // fp32[128]  sc
  static constexpr uint32_t M_META = 1280;  // int[16]
  static constexpr uint32_t M_BAR = 1344;   // 16 mbarriers
  static constexpr uint32_t MISC_GROUP = 1472;
  static constexpr uint32_t BYTES = MISC + NGROUP * MISC_GROUP + 32;
};
// TMEM columns per transform group (group g at 256 g)
constexpr uint32_t TT_G = 0;    // cumulative log decay [r][c] fp32 128
constexpr uint32_t TT_AP = 128; // [A_raw; P_raw] fp32              64
constexpr uint32_t TT_W = 192;  // W'^T fp32                        64

// meta words
enum { MT_DONE = 0, MT_SLOW, MT_N, MT_H, MT_J, MT_L, MT_I, MT_POS, MT_T0LO, MT_T0HI };
// transform mbarriers
enum {
  BT_RAW_FULL = 0, BT_RAW_FREE, BT_CS_GO, BT_CS_FULL, BT_AP_GO, BT_AP_FULL, BT_W_GO, BT_W_FULL, BT_FIN,
  BT_WT_STAGED, BT_WT_READ
};
// state mbarriers
enum {
  BS_A_FULL = 0, BS_A_FREE = 2, BS_B_FULL = 4, BS_B_FREE = 6, BS_S_READY = 8, BS_U_FULL, BS_U_READY, BS_DS_FULL, BS_SP_FREE, BS_O_FULL,
  BS_O_FREE = BS_O_FULL + 2, BS_FIN = BS_O_FREE + 2, BS_G_FULL = BS_FIN + 1, BS_COUNT = BS_G_FULL + 2
};

struct Params {
  int T;            // tokens per batch row, or the packed total with cu
  int H;            // heads
  int N;            // sequences
  int R;            // state CTAs
  const int32_t* cu;
  const void* beta;
  StateIO st;       // initial / final states (dense rows or pool slots)
  __nv_bfloat16* o;
  // producer steps (PROD instantiation): q, k are raw and L2-normalised here;
  // the log-decay tile is the gate projection f, log alpha = -exp(A_log[h]) *
  // softplus(f + dt_bias[h][c])
  const float* A_log;    // [H]
  const float* dt_bias;  // [H][dk]
  // optional output epilogue (gate == nullptr: o is written as computed):
  // o <- o / rms(o) * norm_w * sigmoid(gate), rms over the head's dv values
  const __nv_bfloat16* gate;  // [B, T, H, dv], like o
  const float* norm_w;        // [dv]
  float eps;
  int nring;        // ring slots per state CTA, 2..MAX_RING
  uint8_t* ring;    // R * nring slots
  uint32_t* flags;  // flag_words(R), zero on entry
};

struct Maps {
  CUtensorMap q, k, v, la;
  CUtensorMap o;  // output, box of 64 values x 32 rows
  CUtensorMap g;  // output gate (fused epilogue only), like o
};

// --------------------------------------------------------------------------- helpers
__device__ __forceinline__ void seq_range(const Params& p, int n, int64_t* b, int64_t* e) {
  if (p.cu) {
    *b = p.cu[n];
    *e = p.cu[n + 1];
  } else {
    *b = static_cast<int64_t>(n) * p.T;
    *e = *b + p.T;
  }
}
__device__ __forceinline__ int seq_chunks(const Params& p, int n) {
  int64_t b, e;
  seq_range(p, n, &b, &e);
  return static_cast<int>((e - b + C - 1) / C);
}
__device__ __forceinline__ int stream_len(const Params& p, int i) {
  int len = 0;
  for (int ci = i; ci < p.N * p.H; ci += p.R) len += seq_chunks(p, ci / p.H);
  return len;
}

template <typename TG>
__device__ __forceinline__ float ld_gate(const TG* ptr);
template <>
__device__ __forceinline__ float ld_gate<float>(const float* ptr) { return *ptr; }
template <>
__device__ __forceinline__ float ld_gate<__nv_bfloat16>(const __nv_bfloat16* ptr) { return __bfloat162float(*ptr); }

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void sts128(uint8_t* p, uint4 x) { *reinterpret_cast<uint4*>(p) = x; }
__device__ __forceinline__ void stg128(uint8_t* p, uint4 x) { *reinterpret_cast<uint4*>(p) = x; }
__device__ __forceinline__ float2 bf2f(uint32_t u) {
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(b);
}

// Polls a global counter until it reaches `target` (acquire).  Gives up when
// the kernel-wide abort flag is raised or the wait runs out (then it raises
// the flag itself and records KDA_ERR_TIMEOUT).
__device__ __forceinline__ bool spin_geq(const uint32_t* flag, uint32_t target, uint32_t* gabort,
                                         volatile int* abort_flag) {
  if (ld_acquire_gpu(flag) >= target) return true;
  const long long t0 = clock64();
  for (uint32_t it = 0;; ++it) {
    __nanosleep(64);
    if (ld_acquire_gpu(flag) >= target) return true;
    if ((it & 15u) == 15u) {
      if (*abort_flag || *reinterpret_cast<volatile uint32_t*>(gabort) != 0u) {
        *abort_flag = 1;
        return false;
      }
      if (clock64() - t0 > kWaitCycles) {
        record_error(-8 /* KDA_ERR_TIMEOUT */);
        atomicExch(gabort, 1u);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Element (r, s) of a 64 x 64 fp32 matrix whose 4-float groups are XOR-permuted
// per row, so that 4 or 8 consecutive rows read at one column hit distinct banks.
__device__ __forceinline__ int swzA(int r, int s) { return r * 64 + (s ^ ((((r & 7) ^ ((r >> 3) & 7))) << 2)); }

// ===========================================================================
// transform role: one group of 4 compute warps + a load warp + an MMA warp
// PROD: the producer steps (L2 norm of q and k, the decay gate from its
// projection) run here, on the raw tiles; TG is then bf16.
// ===========================================================================
template <typename TG, bool PROD>
struct Tf {
  using LY = TfLayout<TG>;
  uint8_t* smem;
  uint32_t sbase;
  uint8_t* gb;     // group base
  uint32_t gba;    // group base (shared address)
  uint8_t* misc;
  uint64_t* bars;
  int* meta;
  uint32_t tmem;   // group TMEM base
  int g;

  __device__ Tf(uint8_t* sm, uint32_t tm, int grp) : smem(sm), g(grp) {
    sbase = smem_u32(sm);
    gb = sm + LY::GBASE + grp * LY::GROUP;
    gba = sbase + LY::GBASE + grp * LY::GROUP;
    misc = sm + LY::MISC + grp * LY::MISC_GROUP;
    bars = reinterpret_cast<uint64_t*>(misc + LY::M_BAR);
    meta = reinterpret_cast<int*>(misc + LY::M_META);
    tmem = tm + 256u * grp;
  }
  __device__ float* betas() const { return reinterpret_cast<float*>(misc + LY::M_BETA); }
  __device__ float* gls() const { return reinterpret_cast<float*>(misc + LY::M_GL); }
  __device__ float* scs() const { return reinterpret_cast<float*>(misc + LY::M_SC); }
  // T (fp32, [64][64]) lives in the Qa rows of the [Ka; Qa] tile once A/P is
  // done; its 4-float groups are XOR-permuted per row like A's (tcol()).
  __device__ float* trow(int r) const {
    return reinterpret_cast<float*>(gb + LY::G_KQ + (r < 32 ? 8192 : 24576) + (r & 31) * 256);
  }
  __device__ static int tcol(int r, int s) { return s ^ ((((r & 7) ^ ((r >> 3) & 7))) << 2); }
  __device__ float* amat() const { return reinterpret_cast<float*>(gb + LY::G_KB); }
  // producer: 1/|q_r| at [r], 1/|k_r| at [64 + r] (the upper half of the
  // log-decay tile is dead from the cumsum MMA until the next raw tiles)
  __device__ float* qk_norms() const { return reinterpret_cast<float*>(gb + LY::G_RL + 10240); }
  __device__ void bar() const { named_bar(1 + g, 128); }
  // The cumsum operand is the raw TMA tile unless rows past the chunk end must
  // be zeroed, or fp32 gates (or the producer's log-decay) must be split into
  // bf16 parts first.
  __device__ static bool needs_prep(int L) { return PROD || sizeof(TG) != 2 || L < C; }
  static constexpr bool kSplitGate = PROD || sizeof(TG) != 2;

  // ------------------------------------------------------------ load warp
  __device__ void load_loop(const Maps& maps, const Params& p, int maxlen, volatile int* abort_flag) {
    const int lane = threadIdx.x & 31;
    uint32_t* gflags = p.flags;
    const long long total = static_cast<long long>(p.R) * maxlen;
    int it = 0;
    int prev_si = -1, prev_pos = 0;  // chunk whose -W'^T copy and publication are still due (lane 0)
    int nfinished = 0;
    // Ships the previous chunk's -W'^T tile once the compute warps staged it,
    // waits for every copy of that chunk to land, and publishes its ring slot.
    auto finish_prev = [&]() -> bool {
      if (prev_si < 0) return true;
      const int k = nfinished;
      if (!mbar_wait(&bars[BT_WT_STAGED], k & 1, abort_flag)) return false;
      uint8_t* pslot = p.ring + (static_cast<size_t>(prev_si) * p.nring + (prev_pos % p.nring)) * SLOT;
      bulk_s2g(pslot + R_WT, gb + LY::G_KB, 16384);
      bulk_commit();
      bulk_wait_read<0>();
      mbar_arrive(&bars[BT_WT_READ]);
      bulk_wait_all();
      if (!*abort_flag) {
        fence_proxy_async_global();
        __threadfence();
        st_release_gpu(gflags + F_REC0 + prev_si * F_REC_STRIDE + (prev_pos % p.nring),
                       static_cast<uint32_t>(prev_pos + 1));
      }
      ++nfinished;
      prev_si = -1;
      return true;
    };
    for (;; ++it) {
      // lane 0 decides; every lane takes the same branch
      int stop = 0, done = 0, i = 0, pos = 0, n = 0, h = 0, j = 0, L = 0;
      int64_t t0 = 0;
      if (lane == 0) {
        if (it >= 1 && !mbar_wait(&bars[BT_RAW_FREE], (it - 1) & 1, abort_flag)) stop = 1;
        while (!stop && !done) {
          if (*abort_flag || *reinterpret_cast<volatile uint32_t*>(gflags + F_ABORT) != 0u) {
            *abort_flag = 1;  // the group's other warps unwind at once
            stop = 1;
            break;
          }
          const long long w = atomicAdd(gflags + F_COUNTER, 1u);
          if (w >= total) {
            done = 1;
            break;
          }
          i = static_cast<int>(w % p.R);
          pos = static_cast<int>(w / p.R);
          // walk state CTA i's chains to the chunk at stream position pos
          int rem = pos;
          bool found = false;
          for (int ci = i; ci < p.N * p.H; ci += p.R) {
            const int nc = seq_chunks(p, ci / p.H);
            if (rem < nc) {
              n = ci / p.H;
              h = ci % p.H;
              j = rem;
              found = true;
              break;
            }
            rem -= nc;
          }
          if (!found) continue;  // past the end of this stream
          int64_t sb, se;
          seq_range(p, n, &sb, &se);
          t0 = sb + static_cast<int64_t>(j) * C;
          L = static_cast<int>(se - t0 < C ? se - t0 : C);
          break;
        }
      }
      stop = __shfl_sync(0xffffffffu, stop, 0);
      done = __shfl_sync(0xffffffffu, done, 0);
      if (stop) break;
      if (done) {
        if (lane == 0) {
          meta[MT_DONE] = 1;
          mbar_arrive(&bars[BT_RAW_FULL]);
        }
        ++it;
        break;
      }
      if (lane == 0) {
        meta[MT_DONE] = 0;  // MT_SLOW belongs to the compute warps (the MMA warp may still read it)
        meta[MT_N] = n;
        meta[MT_H] = h;
        meta[MT_J] = j;
        meta[MT_L] = L;
        meta[MT_I] = i;
        meta[MT_POS] = pos;
        meta[MT_T0LO] = static_cast<int>(static_cast<uint64_t>(t0) & 0xffffffffu);
        meta[MT_T0HI] = static_cast<int>(static_cast<uint64_t>(t0) >> 32);
        const int y = static_cast<int>(t0);
        mbar_arrive_expect_tx(&bars[BT_RAW_FULL], 32768 + LY::RL_BYTES + (PROD ? 4 * D : 0));
        // producer: the head's dt_bias row goes where g_last lives later (dead
        // from the previous chunk's C2 on: the raw tiles were released after it)
        if (PROD) bulk_g2s(misc + LY::M_GL, p.dt_bias + static_cast<int64_t>(h) * D, 4 * D, &bars[BT_RAW_FULL]);
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_2d(gb + LY::G_RQ + hf * 8192, &maps.q, h * D + 64 * hf, y, &bars[BT_RAW_FULL]);
          tma_load_2d(gb + LY::G_RK + hf * 8192, &maps.k, h * D + 64 * hf, y, &bars[BT_RAW_FULL]);
        }
        if (sizeof(TG) == 2) {
          for (int hf = 0; hf < 2; ++hf)
            tma_load_2d(gb + LY::G_RL + hf * 8192, &maps.la, h * D + 64 * hf, y, &bars[BT_RAW_FULL]);
        } else {
          for (int qq = 0; qq < 4; ++qq)
            tma_load_2d(gb + LY::G_RL + qq * 8192, &maps.la, h * D + 32 * qq, y, &bars[BT_RAW_FULL]);
        }
        // while this chunk's tiles are in flight, finish the previous chunk
        if (!finish_prev()) stop = 1;
        prev_si = i;
        prev_pos = pos;
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) break;
    }
    if (lane == 0 && !*abort_flag) finish_prev();
    if (lane == 0) bulk_wait_all();  // copies out of shared memory end before the CTA does
    // a load issued for an item that was never consumed must land before exit
    if (lane == 0 && it >= 1) {
      const long long t0 = clock64();
      while (!mbar_try_wait(&bars[BT_RAW_FULL], (it - 1) & 1) && clock64() - t0 < kWaitCycles) {
      }
    }
  }

  // ------------------------------------------------------------- MMA warp
  __device__ void mma_loop(volatile int* abort_flag) {
    constexpr uint32_t id_cs = make_idesc_bf16(128, 128) | IDESC_B_MN;
    constexpr uint32_t id_ap = make_idesc_bf16(128, 64);
    constexpr uint32_t id_w = make_idesc_bf16(128, 64) | IDESC_A_MN;
    const uint32_t Lb = sbase + LY::L;
    int nprep = 0;  // chunks whose cumsum operand the compute warps prepared first
    for (int it = 0;; ++it) {
      if (!mbar_wait(&bars[BT_RAW_FULL], it & 1, abort_flag)) break;
      if (*reinterpret_cast<volatile int*>(&meta[MT_DONE])) break;
      if (needs_prep(meta[MT_L])) {
        if (!mbar_wait(&bars[BT_CS_GO], nprep & 1, abort_flag)) break;
        ++nprep;
      }
      tc_fence_after();
      if (!kSplitGate) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16_ss(tmem + TT_G, make_sdesc_sw128(Lb + kk * 32, 16, 1024),
                      make_sdesc_sw128(gba + LY::G_RL + kk * 2048, 8192, 1024), id_cs, kk > 0);
      } else {
        // log-decay split into bf16 parts (in the KQ and KB areas): three for
        // fp32 gates, two for the producer's (16 significant bits)
#pragma unroll
        for (int t = 0; t < (PROD ? 2 : 3); ++t) {
          const uint32_t base = gba + (t < 2 ? LY::G_KQ + 16384 * t : LY::G_KB);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + TT_G, make_sdesc_sw128(Lb + kk * 32, 16, 1024),
                        make_sdesc_sw128(base + kk * 2048, 8192, 1024), id_cs, (t | kk) != 0);
        }
      }
      mma_commit(&bars[BT_CS_FULL]);
      if (!mbar_wait(&bars[BT_AP_GO], it & 1, abort_flag)) break;
      tc_fence_after();
      if (!*reinterpret_cast<volatile int*>(&meta[MT_SLOW])) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ss(tmem + TT_AP, make_sdesc_sw128(gba + LY::G_KQ + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                      make_sdesc_sw128(gba + LY::G_KB + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_ap, kk > 0);
      }
      mma_commit(&bars[BT_AP_FULL]);
      if (!mbar_wait(&bars[BT_W_GO], it & 1, abort_flag)) break;
      tc_fence_after();
      // W'^T [c][r] = sum_s Ka[s][c] Tb[r][s]  (A = Ka, M/N-major, channel atoms 16 KB apart)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem + TT_W, make_sdesc_sw128(gba + LY::G_KQ + kk * 2048, 16384, 1024),
                    make_sdesc_sw128(gba + LY::G_TB + kk * 32, 16, 1024), id_w, kk > 0);
      mma_commit(&bars[BT_W_FULL]);
    }
    mma_commit(&bars[BT_FIN]);
    const long long t0 = clock64();
    while (!mbar_try_wait(&bars[BT_FIN], 0) && clock64() - t0 < kWaitCycles) {
    }
  }

  // --------------------------------------------------------- compute warps
  __device__ void compute_loop(const Params& p, volatile int* abort_flag) {
    const int gt = threadIdx.x - 128 * g;  // 0..127
    const int q = gt >> 5, lane = gt & 31;
    const int r = 32 * (q & 1) + lane;    // row of the elementwise / cumsum pass
    const int ch = q >> 1;                // channel half
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    uint32_t* gflags = p.flags;
    float* sbeta = betas();
    float* sgl = gls();
    float* ssc = scs();
    for (int it = 0;; ++it) {
      // one decision for the whole group (its named barriers must stay matched):
      // stop on completion or abort; inside the body a failed wait only raises
      // the abort flag, and every barrier is still reached.
      const bool got = mbar_wait_warp(&bars[BT_RAW_FULL], it & 1, abort_flag);
      const bool fin = got && *reinterpret_cast<volatile int*>(&meta[MT_DONE]) != 0;
      if (named_bar_or(1 + g, 128, !got || fin || *abort_flag)) {
        if (gt == 0) bulk_wait_all();  // copies out of shared memory end before the CTA does
        break;
      }
      const int L = meta[MT_L];
      const int si = meta[MT_I];
      const int pos = meta[MT_POS];
      const int hh = meta[MT_H];
      if (gt == 0) {
        // this chunk's ring slot must have been copied out by its state CTA
        if (pos + 1 - p.nring > 0)
          spin_geq(gflags + F_REC0 + si * F_REC_STRIDE + F_CONSUMED, static_cast<uint32_t>(pos + 1 - p.nring),
                   gflags + F_ABORT, abort_flag);
      }
      const int64_t t0 = static_cast<int64_t>((static_cast<uint64_t>(static_cast<uint32_t>(meta[MT_T0HI])) << 32) |
                                              static_cast<uint32_t>(meta[MT_T0LO]));
      uint8_t* slot = p.ring + (static_cast<size_t>(si) * p.nring + (pos % p.nring)) * SLOT;
      // beta of this chunk (rows >= L are zero); the load overlaps the cumsum
      // MMA, and the group owns its copy (the load warp moves on to the next
      // chunk as soon as the raw tiles are released)
      const float beta_r = gt < L ? ld_gate(static_cast<const TG*>(p.beta) + (t0 + gt) * p.H + hh) : 0.f;

      // the previous chunk's -W'^T staging (KB area) must have been read before
      // anything here writes that area
      if (it >= 1) mbar_wait_warp(&bars[BT_WT_READ], (it - 1) & 1, abort_flag);

      // ---- C1: prepare the cumsum operand (when the raw tile is not usable) ----
      if (!needs_prep(L)) {
      } else if (PROD) {
        // log alpha = -exp(A_log[h]) * softplus(f + dt_bias[h][c]) in fp32 from
        // the bf16 tile of f: softplus(x) = ln 2 * log2(1 + 2^(x log2 e)) on the
        // MUFU unit (x itself beyond 15); split into hi + lo bf16 tiles
        const float nrate = -__expf(p.A_log[hh]);
        const float nrate_ln2 = nrate * 0.69314718f;
        const float* bias = sgl;  // this head's dt_bias, staged by the load warp
#pragma unroll 2
        for (int jj = 0; jj < 8; ++jj) {
          const int c0 = 64 * ch + 8 * jj;
          const uint4 w = lds128(gb + LY::G_RL + ch * 8192 + sw128(r, jj));
          const uint32_t f4[4] = {w.x, w.y, w.z, w.w};
          const float4 ba = *reinterpret_cast<const float4*>(bias + c0);
          const float4 bb = *reinterpret_cast<const float4*>(bias + c0 + 4);
          const float b8[8] = {ba.x, ba.y, ba.z, ba.w, bb.x, bb.y, bb.z, bb.w};
          uint32_t pk[2][4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 fx = bf2f(f4[u]);
            const float x0 = fx.x + b8[2 * u], x1 = fx.y + b8[2 * u + 1];
            float a0 = x0 > 15.f ? nrate * x0 : nrate_ln2 * lg2_approx(1.f + ex2_approx(x0 * kLog2e));
            float a1 = x1 > 15.f ? nrate * x1 : nrate_ln2 * lg2_approx(1.f + ex2_approx(x1 * kLog2e));
            if (r >= L) a0 = a1 = 0.f;
            const float h0 = __bfloat162float(__float2bfloat16_rn(a0)), h1 = __bfloat162float(__float2bfloat16_rn(a1));
            pk[0][u] = pack_bf16(h0, h1);
            pk[1][u] = pack_bf16(a0 - h0, a1 - h1);
          }
          sts128(gb + LY::G_KQ + ch * 8192 + sw128(r, jj), make_uint4(pk[0][0], pk[0][1], pk[0][2], pk[0][3]));
          sts128(gb + LY::G_KQ + 16384 + ch * 8192 + sw128(r, jj), make_uint4(pk[1][0], pk[1][1], pk[1][2], pk[1][3]));
        }
      } else if (sizeof(TG) == 2) {
        if (L < C) {
          for (int e = gt; e < (C - L) * 16; e += 128) {
            const int rr = L + (e >> 4), hf = (e >> 3) & 1, jj = e & 7;
            sts128(gb + LY::G_RL + hf * 8192 + sw128(rr, jj), make_uint4(0u, 0u, 0u, 0u));
          }
        }
      } else {
        // split fp32 log-decay into hi + mid + lo bf16 tiles ([s][c], MN-major B)
#pragma unroll 1
        for (int jj = 0; jj < 8; ++jj) {
          const int c0 = 64 * ch + 8 * jj;
          float x[8];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int c = c0 + 4 * u;
            const uint4 w = lds128(gb + LY::G_RL + (c >> 5) * 8192 + sw128(r, (c & 31) >> 2));
            x[4 * u + 0] = __uint_as_float(w.x);
            x[4 * u + 1] = __uint_as_float(w.y);
            x[4 * u + 2] = __uint_as_float(w.z);
            x[4 * u + 3] = __uint_as_float(w.w);
          }
          uint32_t pk[3][4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float a0 = r < L ? x[2 * u] : 0.f, a1 = r < L ? x[2 * u + 1] : 0.f;
            const float h0 = __bfloat162float(__float2bfloat16_rn(a0)), h1 = __bfloat162float(__float2bfloat16_rn(a1));
            const float m0 = __bfloat162float(__float2bfloat16_rn(a0 - h0));
            const float m1 = __bfloat162float(__float2bfloat16_rn(a1 - h1));
            pk[0][u] = pack_bf16(h0, h1);
            pk[1][u] = pack_bf16(m0, m1);
            pk[2][u] = pack_bf16(a0 - h0 - m0, a1 - h1 - m1);
          }
#pragma unroll
          for (int t = 0; t < 3; ++t) {
            uint8_t* base = gb + (t < 2 ? LY::G_KQ + 16384 * t : LY::G_KB);
            sts128(base + ch * 8192 + sw128(r, jj), make_uint4(pk[t][0], pk[t][1], pk[t][2], pk[t][3]));
          }
        }
      }
      if (needs_prep(L)) {
        fence_proxy_async_smem();
        bar();
        if (gt == 0) mbar_arrive(&bars[BT_CS_GO]);
      }

      // ---- C2: cumulative decay -> scaled tiles ---------------------------------
      if (gt < C) sbeta[gt] = beta_r;  // published by the barriers below
      // producer: |q_r|^2 and |k_r|^2 over this thread's channel half while the
      // cumsum MMA runs; the halves meet in the upper half of the log-decay
      // tile (consumed by C1), read after the barriers below
      float sq = 0.f, sk = 0.f;
      if constexpr (PROD) {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const uint4 kw = lds128(gb + LY::G_RK + ch * 8192 + sw128(r, jj));
          const uint4 qw = lds128(gb + LY::G_RQ + ch * 8192 + sw128(r, jj));
          const uint32_t kk4[4] = {kw.x, kw.y, kw.z, kw.w}, qq4[4] = {qw.x, qw.y, qw.z, qw.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 kx = bf2f(kk4[u]), qx = bf2f(qq4[u]);
            sk = fmaf(kx.x, kx.x, fmaf(kx.y, kx.y, sk));
            sq = fmaf(qx.x, qx.x, fmaf(qx.y, qx.y, sq));
          }
        }
        reinterpret_cast<float2*>(gb + LY::G_RL + 9216)[ch * 64 + r] = make_float2(sq, sk);
      }
      mbar_wait_warp(&bars[BT_CS_FULL], it & 1, abort_flag);
      tc_fence_after();
      float g2[64];
      {
        float x[32];
        tmem_ld32(tmem + lane_off + TT_G + 64 * ch, x);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) g2[u] = x[u] * kLog2e;
        tmem_ld32(tmem + lane_off + TT_G + 64 * ch + 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) g2[32 + u] = x[u] * kLog2e;
      }
      bool steep = false;  // this thread holds row 63 and a channel decays beyond the factorised range
      if ((q & 1) && lane == 31) {
#pragma unroll
        for (int u = 0; u < 64; ++u) {
          sgl[64 * ch + u] = g2[u];
          steep = steep || (-g2[u] > kSpan2);
        }
      }
      const bool slow = named_bar_or(1 + g, 128, steep);
      {
        // per channel: sc = 2^{g_last/2} (1 on the exact path), gamma_C = 2^{g_last}
        const float gl = sgl[gt];
        const float sc = slow ? 1.f : ex2_approx(0.5f * gl);
        ssc[gt] = sc;
        float* vec = reinterpret_cast<float*>(slot + R_VEC);
        vec[gt] = sc;
        vec[128 + gt] = ex2_approx(gl);
      }
      bar();
      // producer: 1 / |q_r| and 1 / |k_r| from both halves' partial sums; the
      // exact path reads every row's factors (published by its own barrier)
      float rq = 1.f, rk = 1.f;
      if constexpr (PROD) {
        const float2 o = reinterpret_cast<const float2*>(gb + LY::G_RL + 9216)[(ch ^ 1) * 64 + r];
        rq = rsqrtf(sq + o.x + kQKNormEps);
        rk = rsqrtf(sk + o.y + kQKNormEps);
        if (ch == 0) {
          float* rn = qk_norms();
          rn[r] = rq;
          rn[64 + r] = rk;
        }
      }
      // q_r . k_r over this thread's channel half, in fp32 from the raw bf16
      // inputs: the diagonal of P, where the decay factors cancel exactly.  The
      // bf16-rounded scaled operands would lose it to cancellation when q_r and
      // k_r are nearly orthogonal (it is the whole output of a token that
      // starts from a zero state).
      float pdiag = 0.f;
      if (!slow) {
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int c0 = 64 * ch + 8 * jj;
          const float4 gla = *reinterpret_cast<const float4*>(sgl + c0);
          const float4 glb = *reinterpret_cast<const float4*>(sgl + c0 + 4);
          const float4 sca = *reinterpret_cast<const float4*>(ssc + c0);
          const float4 scb = *reinterpret_cast<const float4*>(ssc + c0 + 4);
          const float rf8[8] = {0.5f * gla.x, 0.5f * gla.y, 0.5f * gla.z, 0.5f * gla.w,
                                0.5f * glb.x, 0.5f * glb.y, 0.5f * glb.z, 0.5f * glb.w};
          const float sc8[8] = {sca.x, sca.y, sca.z, sca.w, scb.x, scb.y, scb.z, scb.w};
          uint4 kw = lds128(gb + LY::G_RK + ch * 8192 + sw128(r, jj));
          uint4 qw = lds128(gb + LY::G_RQ + ch * 8192 + sw128(r, jj));
          if (r >= L) kw = qw = make_uint4(0u, 0u, 0u, 0u);
          const uint32_t kk4[4] = {kw.x, kw.y, kw.z, kw.w}, qq4[4] = {qw.x, qw.y, qw.z, qw.w};
          uint32_t ka[4], qa[4], kb[4], kt[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float2 kx = bf2f(kk4[u]), qx = bf2f(qq4[u]);
            if constexpr (PROD) {
              kx.x *= rk, kx.y *= rk;
              qx.x *= rq, qx.y *= rq;
            }
            pdiag = fmaf(qx.x, kx.x, fmaf(qx.y, kx.y, pdiag));
            const float rf0 = rf8[2 * u], rf1 = rf8[2 * u + 1];
            const float x0 = g2[8 * jj + 2 * u], x1 = g2[8 * jj + 2 * u + 1];
            const float d0 = x0 - rf0, d1 = x1 - rf1;
            const float e10 = ex2_approx(d0), e11 = ex2_approx(d1);
            const float e20 = ex2_approx(-d0), e21 = ex2_approx(-d1);
            ka[u] = pack_bf16(kx.x * e10, kx.y * e11);
            qa[u] = pack_bf16(qx.x * e10, qx.y * e11);
            const float b0 = kx.x * e20, b1 = kx.y * e21;
            kb[u] = pack_bf16(b0, b1);
            kt[u] = pack_bf16(b0 * sc8[2 * u], b1 * sc8[2 * u + 1]);
          }
          sts128(gb + LY::G_KQ + ch * 16384 + sw128(r, jj), make_uint4(ka[0], ka[1], ka[2], ka[3]));
          sts128(gb + LY::G_KQ + ch * 16384 + sw128(64 + r, jj), make_uint4(qa[0], qa[1], qa[2], qa[3]));
          sts128(gb + LY::G_KB + ch * 8192 + sw128(r, jj), make_uint4(kb[0], kb[1], kb[2], kb[3]));
          // Kt replaces the raw k chunk this thread just read (ring layout)
          sts128(gb + LY::G_RK + ch * 8192 + sw128(r, jj), make_uint4(kt[0], kt[1], kt[2], kt[3]));
        }
        // the first channel half hands its partial to the thread of the second
        // half that writes row r of P (same r), through the upper half of the
        // log-decay tile: dead since the cumsum MMA completed, not reloaded
        // before this chunk's raw tiles are released, and not under P
        if (ch == 0) reinterpret_cast<float*>(gb + LY::G_RL + 8192)[r] = pdiag;
      } else {
        // ---- exact path: A and P term by term from g (fp32, in the KQ area) ------
        float* G = reinterpret_cast<float*>(gb + LY::G_KQ);
#pragma unroll
        for (int u = 0; u < 64; u += 4)
          *reinterpret_cast<float4*>(G + r * 128 + 64 * ch + u) = make_float4(g2[u], g2[u + 1], g2[u + 2], g2[u + 3]);
        bar();
        const uint8_t* RK = gb + LY::G_RK;
        const uint8_t* RQ = gb + LY::G_RQ;
        auto kval = [&](const uint8_t* tile, int row, int c) -> float {
          const uint16_t raw = *reinterpret_cast<const uint16_t*>(tile + (c >> 6) * 8192 + sw128(row, (c & 63) >> 3) +
                                                                  (c & 7) * 2);
          return row < L ? __bfloat162float(__ushort_as_bfloat16(raw)) : 0.f;
        };
        float* Af = amat();
#pragma unroll 1
        for (int e = gt; e < C * C; e += 128) {
          const int ar = e >> 6, as = e & 63;
          float a = 0.f, pp = 0.f;
          if (as <= ar) {
#pragma unroll 4
            for (int c = 0; c < D; ++c) {
              const float ex = ex2_approx(G[ar * 128 + c] - G[as * 128 + c]);
              const float kse = kval(RK, as, c) * ex;
              a += kval(RK, ar, c) * kse;
              pp += kval(RQ, ar, c) * kse;
            }
          }
          if constexpr (PROD) {
            const float* rn = qk_norms();
            a *= rn[64 + ar] * rn[64 + as];
            pp *= rn[ar] * rn[64 + as];
          }
          Af[swzA(ar, as)] = as < ar ? sbeta[ar] * a : 0.f;
          *reinterpret_cast<__nv_bfloat16*>(gb + LY::G_RL + sw128(ar, as >> 3) + (as & 7) * 2) =
              __float2bfloat16_rn(pp);
        }
        bar();  // g is dead; Ka / Qa overwrite it
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int c0 = 64 * ch + 8 * jj;
          uint4 kw = lds128(gb + LY::G_RK + ch * 8192 + sw128(r, jj));
          uint4 qw = lds128(gb + LY::G_RQ + ch * 8192 + sw128(r, jj));
          if (r >= L) kw = qw = make_uint4(0u, 0u, 0u, 0u);
          const uint32_t kk4[4] = {kw.x, kw.y, kw.z, kw.w}, qq4[4] = {qw.x, qw.y, qw.z, qw.w};
          uint32_t ka[4], qa[4], kt[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int c = c0 + 2 * u;
            float2 kx = bf2f(kk4[u]), qx = bf2f(qq4[u]);
            if constexpr (PROD) {
              kx.x *= rk, kx.y *= rk;
              qx.x *= rq, qx.y *= rq;
            }
            const float x0 = g2[8 * jj + 2 * u], x1 = g2[8 * jj + 2 * u + 1];
            const float gm0 = ex2_approx(x0), gm1 = ex2_approx(x1);
            const float ps0 = ex2_approx(sgl[c] - x0), ps1 = ex2_approx(sgl[c + 1] - x1);
            ka[u] = pack_bf16(kx.x * gm0, kx.y * gm1);
            qa[u] = pack_bf16(qx.x * gm0, qx.y * gm1);
            kt[u] = pack_bf16(kx.x * ps0, kx.y * ps1);
          }
          sts128(gb + LY::G_KQ + ch * 16384 + sw128(r, jj), make_uint4(ka[0], ka[1], ka[2], ka[3]));
          sts128(gb + LY::G_KQ + ch * 16384 + sw128(64 + r, jj), make_uint4(qa[0], qa[1], qa[2], qa[3]));
          sts128(gb + LY::G_RK + ch * 8192 + sw128(r, jj), make_uint4(kt[0], kt[1], kt[2], kt[3]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      bar();
      if (gt == 0) {
        meta[MT_SLOW] = slow ? 1 : 0;
        mbar_arrive(&bars[BT_AP_GO]);
        // Qa (the lower half of each [Ka; Qa] atom) and Kt go to the ring slot
        bulk_s2g(slot + R_QA, gb + LY::G_KQ + 8192, 8192);
        bulk_s2g(slot + R_QA + 8192, gb + LY::G_KQ + 16384 + 8192, 8192);
        bulk_s2g(slot + R_KT, gb + LY::G_RK, 16384);
        bulk_commit();
      }

      // ---- C3: A / P epilogue -------------------------------------------------------
      mbar_wait_warp(&bars[BT_AP_FULL], it & 1, abort_flag);
      tc_fence_after();
      if (!slow) {
        float x[64];
        {
          float t[32];
          tmem_ld32(tmem + lane_off + TT_AP, t);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) x[u] = t[u];
          tmem_ld32(tmem + lane_off + TT_AP + 32, t);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 32; ++u) x[32 + u] = t[u];
        }
        if (q < 2) {
          const int ar = 32 * q + lane;
          const float br = sbeta[ar];
          float* Af = amat();
#pragma unroll
          for (int s4 = 0; s4 < 16; ++s4) {
            float4 w;
            w.x = 4 * s4 + 0 < ar ? br * x[4 * s4 + 0] : 0.f;
            w.y = 4 * s4 + 1 < ar ? br * x[4 * s4 + 1] : 0.f;
            w.z = 4 * s4 + 2 < ar ? br * x[4 * s4 + 2] : 0.f;
            w.w = 4 * s4 + 3 < ar ? br * x[4 * s4 + 3] : 0.f;
            *reinterpret_cast<float4*>(Af + swzA(ar, 4 * s4)) = w;
          }
        } else {
          const int rp = 32 * (q - 2) + lane;  // == r of this thread (channel half 1)
          const float dg = pdiag + reinterpret_cast<const float*>(gb + LY::G_RL + 8192)[rp];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            uint32_t pk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int s0 = 8 * jj + 2 * u;
              const float p0 = s0 < rp ? x[s0] : (s0 == rp ? dg : 0.f);
              const float p1 = s0 + 1 < rp ? x[s0 + 1] : (s0 + 1 == rp ? dg : 0.f);
              pk[u] = pack_bf16(p0, p1);
            }
            sts128(gb + LY::G_RL + sw128(rp, jj), make_uint4(pk[0], pk[1], pk[2], pk[3]));
          }
        }
      }
      fence_proxy_async_smem();
      bar();
      if (gt == 0) {
        bulk_s2g(slot + R_PP, gb + LY::G_RL, 8192);
        bulk_commit();
      }

      // ---- C4: T = (I + A)^-1, blocked forward substitution (fp32) ---------------
      invert(sbeta);
      // Tb = T Diag(beta) -> bf16 [r][s] (local MMA operand, shipped to the ring
      // slot); 8 threads share a row, one 16-byte chunk of 8 columns each
      {
        const int jq = gt & 7;
        const int s0 = 8 * jq;
        const float4 b0 = *reinterpret_cast<const float4*>(sbeta + s0);
        const float4 b1 = *reinterpret_cast<const float4*>(sbeta + s0 + 4);
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int tr = 16 * pass + (gt >> 3);
          uint32_t pk[4] = {0u, 0u, 0u, 0u};
          if ((s0 >> 4) <= (tr >> 4)) {
            const float* Tr = trow(tr);
            const float4 t0 = *reinterpret_cast<const float4*>(Tr + tcol(tr, s0));
            const float4 t1 = *reinterpret_cast<const float4*>(Tr + tcol(tr, s0 + 4));
            pk[0] = pack_bf16(t0.x * b0.x, t0.y * b0.y);
            pk[1] = pack_bf16(t0.z * b0.z, t0.w * b0.w);
            pk[2] = pack_bf16(t1.x * b1.x, t1.y * b1.y);
            pk[3] = pack_bf16(t1.z * b1.z, t1.w * b1.w);
          }
          sts128(gb + LY::G_TB + sw128(tr, jq), make_uint4(pk[0], pk[1], pk[2], pk[3]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      bar();
      if (gt == 0) {
        mbar_arrive(&bars[BT_W_GO]);
        bulk_s2g(slot + R_TB, gb + LY::G_TB, 8192);
        bulk_commit();
      }

      // ---- C5: -W'^T -> ring slot, then publish --------------------------------------
      mbar_wait_warp(&bars[BT_W_FULL], it & 1, abort_flag);
      tc_fence_after();
      {
        const int c = 32 * q + lane;
        float x[32];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          tmem_ld32(tmem + lane_off + TT_W + 32 * hf, x);
          tmem_wait_ld();
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            uint32_t pk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) pk[u] = pack_bf16(-x[8 * j4 + 2 * u], -x[8 * j4 + 2 * u + 1]);
            sts128(gb + LY::G_KB + sw128(c, 4 * hf + j4), make_uint4(pk[0], pk[1], pk[2], pk[3]));
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      bar();
      if (gt == 0) {
        // this thread's copies (Qa, Kt, P, Tb) have landed; the load warp ships
        // -W'^T and publishes the slot
        bulk_wait_all();
        fence_proxy_async_global();
        mbar_arrive(&bars[BT_WT_STAGED]);
      }
    }
  }

  // T = (I + A)^-1 for the strictly lower-triangular A (fp32, swizzled rows in
  // the KB area), written to trow().  Diagonal 16 x 16 blocks by row-wise
  // forward substitution; then block levels d = 1, 2, 3:
  //   T_IJ = -T_II sum_{K=J}^{I-1} A_IK T_KJ      (I - J = d)
  // Block indices are compile-time, so every shared-memory offset except the
  // thread's own row / column is an immediate.
  __device__ static int swz4(int r) { return (((r & 7) ^ ((r >> 3) & 7))) << 2; }

  // X_b[i][j0, j0+1] = sum_{K=J}^{I-1} A_IK[i][:] T_KJ[:][j0, j0+1]
  template <int I, int J>
  __device__ __forceinline__ void level_x(float* X, int b, int i, int j0) const {
    const float* Ar = amat() + (16 * I + i) * 64;
    const int sa = swz4(16 * I + i);
    float a0 = 0.f, a1 = 0.f, c0 = 0.f, c1 = 0.f;
#pragma unroll
    for (int K = J; K < I; ++K) {
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4) {
        const float4 av = *reinterpret_cast<const float4*>(Ar + ((16 * K + 4 * g4) ^ sa));
        const float aa[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int rt = 16 * K + 4 * g4 + u;
          const float2 tv = *reinterpret_cast<const float2*>(trow(rt) + tcol(rt, 16 * J + j0));
          if (u & 1) {
            c0 += aa[u] * tv.x;
            c1 += aa[u] * tv.y;
          } else {
            a0 += aa[u] * tv.x;
            a1 += aa[u] * tv.y;
          }
        }
      }
    }
    *reinterpret_cast<float2*>(X + (b * 16 + i) * 16 + j0) = make_float2(a0 + c0, a1 + c1);
  }
  // T_IJ[i][j0, j0+1] = -T_II[i][:] X_b[:][j0, j0+1]
  template <int I, int J>
  __device__ __forceinline__ void level_t(const float* X, int b, int i, int j0) {
    const int rt = 16 * I + i;
    float* Tr = trow(rt);
    const int st = swz4(rt);
    float a0 = 0.f, a1 = 0.f, c0 = 0.f, c1 = 0.f;
#pragma unroll
    for (int g4 = 0; g4 < 4; ++g4) {
      const float4 tv = *reinterpret_cast<const float4*>(Tr + ((16 * I + 4 * g4) ^ st));
      const float tt[4] = {tv.x, tv.y, tv.z, tv.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 xv = *reinterpret_cast<const float2*>(X + (b * 16 + 4 * g4 + u) * 16 + j0);
        if (u & 1) {
          c0 += tt[u] * xv.x;
          c1 += tt[u] * xv.y;
        } else {
          a0 += tt[u] * xv.x;
          a1 += tt[u] * xv.y;
        }
      }
    }
    *reinterpret_cast<float2*>(Tr + ((16 * J + j0) ^ st)) = make_float2(-(a0 + c0), -(a1 + c1));
  }

  __device__ void invert(const float* sbeta) {
    const int gt = threadIdx.x - 128 * g;
    const float* Af = amat();
    float* X = reinterpret_cast<float*>(gb + LY::G_TB);  // scratch, [3][16][16]
    float x[16];
    if (gt < 64) {
      // column jc of T_II: x_i = delta_ij - sum_{m<i} A_II[i][m] x_m, one row at a time
      const int I = gt >> 4, jc = gt & 15;
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) {
        const int ra = 16 * I + ii;
        const float* Ar = Af + ra * 64;
        const int sa = swz4(ra);
        float acc0 = ii == jc ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
          if (4 * g4 < ii) {
            const float4 av = *reinterpret_cast<const float4*>(Ar + ((16 * I + 4 * g4) ^ sa));
            const float aa[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (4 * g4 + u < ii) {
                if (u & 1)
                  acc1 -= aa[u] * x[4 * g4 + u];
                else
                  acc0 -= aa[u] * x[4 * g4 + u];
              }
            }
          }
        }
        x[ii] = acc0 + acc1;
      }
    }
    // T overwrites Qa: the copies out of shared memory (Qa, Kt, P) must have
    // read their sources first; then the raw tiles are free for the next
    // chunk.  The wait overlaps the diagonal solves above.
    if (gt == 0) {
      bulk_wait_read<0>();
      mbar_arrive(&bars[BT_RAW_FREE]);
    }
    bar();
    if (gt < 64) {
      const int I = gt >> 4, jc = gt & 15;
#pragma unroll
      for (int ii = 0; ii < 16; ++ii) trow(16 * I + ii)[tcol(16 * I + ii, 16 * I + jc)] = x[ii];
    }
    bar();
    const int i = gt >> 3, j0 = 2 * (gt & 7);  // each thread: row i, columns j0, j0+1 of a 16 x 16 block
    level_x<1, 0>(X, 0, i, j0);
    level_x<2, 1>(X, 1, i, j0);
    level_x<3, 2>(X, 2, i, j0);
    bar();
    level_t<1, 0>(X, 0, i, j0);
    level_t<2, 1>(X, 1, i, j0);
    level_t<3, 2>(X, 2, i, j0);
    bar();
    level_x<2, 0>(X, 0, i, j0);
    level_x<3, 1>(X, 1, i, j0);
    bar();
    level_t<2, 0>(X, 0, i, j0);
    level_t<3, 1>(X, 1, i, j0);
    bar();
    level_x<3, 0>(X, 0, i, j0);
    bar();
    level_t<3, 0>(X, 0, i, j0);
    bar();
  }
};

// ===========================================================================
// state role
// ===========================================================================
struct StateWalk {
  int ci, nc;
  int64_t sb, se;
  __device__ bool next(const Params& p) {
    ci += p.R;
    if (ci >= p.N * p.H) return false;
    seq_range(p, ci / p.H, &sb, &se);
    nc = static_cast<int>((se - sb + C - 1) / C);
    return true;
  }
};

__device__ __forceinline__ void state_load_loop(uint8_t* smem, const Maps& maps, const Params& p, uint64_t* bars,
                                                volatile int* abort_flag) {
  const int i = blockIdx.x;
  uint32_t* gflags = p.flags;
  const uint32_t* ready = gflags + F_REC0 + i * F_REC_STRIDE;
  uint32_t* consumed = gflags + F_REC0 + i * F_REC_STRIDE + F_CONSUMED;
  int pos = 0;
  bool ok = true;
  StateWalk w{i - p.R, 0, 0, 0};
  while (ok && w.next(p)) {
    const int h = w.ci % p.H;
    for (int j = 0; j < w.nc; ++j, ++pos) {
      const int s = pos & 1;
      const uint32_t par = ((pos - 2) >> 1) & 1;
      // part A and V into buffer s once position pos-2 has finished with them
      if (pos >= 2 && !mbar_wait(&bars[BS_A_FREE + s], par, abort_flag)) { ok = false; break; }
      if (!spin_geq(ready + (pos % p.nring), static_cast<uint32_t>(pos + 1), gflags + F_ABORT, abort_flag)) {
        ok = false;
        break;
      }
      fence_proxy_async_global();
      const int64_t t0 = w.sb + static_cast<int64_t>(j) * C;
      const uint8_t* src = p.ring + (static_cast<size_t>(i) * p.nring + (pos % p.nring)) * SLOT;
      mbar_arrive_expect_tx(&bars[BS_A_FULL + s], SLOT_A + 16384);
      bulk_g2s(smem + ST_A + s * SLOT_A, src, SLOT_A, &bars[BS_A_FULL + s]);
      for (int hf = 0; hf < 2; ++hf)
        tma_load_2d(smem + ST_V + s * 16384 + hf * 8192, &maps.v, h * D + 64 * hf, static_cast<int>(t0),
                    &bars[BS_A_FULL + s]);
      // part B
      if (pos >= 2 && !mbar_wait(&bars[BS_B_FREE + s], par, abort_flag)) { ok = false; ++pos; break; }
      mbar_arrive_expect_tx(&bars[BS_B_FULL + s], SLOT_B);
      bulk_g2s(smem + ST_B + s * SLOT_B, src + SLOT_A, SLOT_B, &bars[BS_B_FULL + s]);
      // the previous position's copies have landed: its ring slot may be reused
      if (pos >= 1) {
        const int pp = pos - 1;
        if (!mbar_wait(&bars[BS_A_FULL + (pp & 1)], (pp >> 1) & 1, abort_flag) ||
            !mbar_wait(&bars[BS_B_FULL + (pp & 1)], (pp >> 1) & 1, abort_flag)) {
          ok = false;
          ++pos;
          break;
        }
        fence_proxy_async_global();
        st_release_gpu(consumed, static_cast<uint32_t>(pos));
      }
    }
  }
  // drain: copies still landing in shared memory must finish before exit
  for (int pp = pos - 2 < 0 ? 0 : pos - 2; pp < pos; ++pp) {
    const long long t0 = clock64();
    while (!mbar_try_wait(&bars[BS_A_FULL + (pp & 1)], (pp >> 1) & 1) && clock64() - t0 < kWaitCycles) {
    }
    while (!mbar_try_wait(&bars[BS_B_FULL + (pp & 1)], (pp >> 1) & 1) && clock64() - t0 < kWaitCycles) {
    }
  }
}

// The MMAs of one position (slot s = b = position parity), in issue order:
//   U^T  = V^T Tb^T            (state-independent, first)
//   U^T += S'^T (-W'^T)        -> U_FULL
//   dS^T = U^T Kt              -> DS_FULL   (the chain: the next S waits on it)
//   O    = Qa S'               -> SP_FREE   (S' may be overwritten after it)
//   O   += P U                 -> O_FULL, B_FREE
// O is produced off the chain, after dS.  Its products are issued with M = 128
// and an A operand that starts 64 rows before Qa (resp. P) in shared memory,
// so that the 64 output rows land in TMEM lanes 64-127, where the two output
// warps (10 and 11) can read them; lanes 0-63 receive unused products.
__device__ __forceinline__ void state_mma_loop(uint32_t sbase, uint32_t tmem, const Params& p, uint64_t* bars,
                                               volatile int* abort_flag) {
  constexpr uint32_t id_uv = make_idesc_bf16(128, 64) | IDESC_A_MN;
  constexpr uint32_t id_us = make_idesc_bf16(128, 64) | IDESC_B_MN;
  constexpr uint32_t id_o = make_idesc_bf16(128, 128);
  constexpr uint32_t id_ds = make_idesc_bf16(128, 128) | IDESC_B_MN;
  const int i = blockIdx.x;
  int pos = 0;
  bool ok = true;
  StateWalk w{i - p.R, 0, 0, 0};
  while (ok && w.next(p)) {
    for (int j = 0; j < w.nc; ++j, ++pos) {
      const int s = pos & 1, b = pos & 1;
      const uint32_t sa = sbase + ST_A + s * SLOT_A;          // part A of this position
      const uint32_t sb2 = sbase + ST_B + s * SLOT_B - SLOT_A;  // part B, addressed with ring offsets
      const uint32_t vt = sbase + ST_V + s * 16384;
      if (!mbar_wait(&bars[BS_A_FULL + s], (pos >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      // U^T = V^T Tb^T
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem + TS_U, make_sdesc_sw128(vt + kk * 2048, 8192, 1024),
                    make_sdesc_sw128(sa + R_TB + kk * 32, 16, 1024), id_uv, kk > 0);
      if (!mbar_wait(&bars[BS_S_READY], pos & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      // U^T += S'^T (-W'^T)
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tmem + TS_U, make_sdesc_sw128(sbase + ST_S + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                    make_sdesc_sw128(sa + R_WT + kk * 2048, 8192, 1024), id_us, 1);
#ifdef KDA_TEST_HOOKS
      if (!(g_test_skip_commit != 0 && blockIdx.x == 0 && pos == 0))
#endif
        mma_commit(&bars[BS_U_FULL]);
      if (!mbar_wait(&bars[BS_U_READY], pos & 1, abort_flag)) { ok = false; break; }
      // the state warps arrive on U_READY after their last read of the scales:
      // part A frees once the MMAs issued so far have read it
      mma_commit(&bars[BS_A_FREE + s]);
      if (!mbar_wait(&bars[BS_B_FULL + s], (pos >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      // dS^T = U^T Kt
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem + TS_DS, make_sdesc_sw128(sbase + ST_U + kk * 32, 16, 1024),
                    make_sdesc_sw128(sb2 + R_KT + kk * 2048, 8192, 1024), id_ds, kk > 0);
      mma_commit(&bars[BS_DS_FULL]);
      // O = Qa S'  (buffer b, free once position pos-2 was read out; S'^T [v][c]
      // is the K-major B operand; the A operand's rows start 8 KB = 64 rows
      // before each 64-channel atom of Qa)
      if (pos >= 2 && !mbar_wait(&bars[BS_O_FREE + b], ((pos - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16_ss(tmem + TS_O + 128 * b,
                    make_sdesc_sw128(sb2 + R_QA - 8192 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                    make_sdesc_sw128(sbase + ST_S + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), id_o, kk > 0);
      mma_commit(&bars[BS_SP_FREE]);
      // O += P U  (U^T [v][r] is the K-major B operand; the A rows start 64 rows before P)
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem + TS_O + 128 * b, make_sdesc_sw128(sb2 + R_PP - 8192 + kk * 32, 16, 1024),
                    make_sdesc_sw128(sbase + ST_U + kk * 32, 16, 1024), id_o, 1);
      mma_commit(&bars[BS_O_FULL + b]);
      mma_commit(&bars[BS_B_FREE + s]);
    }
    if (!ok) break;
  }
  mma_commit(&bars[BS_FIN]);
  const long long t0 = clock64();
  while (!mbar_try_wait(&bars[BS_FIN], 0) && clock64() - t0 < kWaitCycles) {
  }
}

// Waits, with a bound and regardless of the abort flag, for a tile load in
// flight into shared memory to land (a CTA must not end with one pending).
__device__ __forceinline__ void drain_tile(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 < kWaitCycles) {
  }
}

// Warps 10 and 11 write O: warp 10 + u holds output rows 32 u + lane of a
// chunk (TMEM lanes 64 + 32 u + lane), 128 values each.  Each warp stages its
// 32 x 128 block as bf16 in shared memory and stores it with two tensor
// stores when all its rows belong to the sequence, else row by row.
//
// GATED: the output epilogue of the Kimi Linear layer, o <- o / rms(o) *
// norm_w * sigmoid(gate) per (token, head) row.  The warp's 32 x 128 gate
// tile comes by TMA into the staging block (where the outputs go, in the
// same swizzled layout) while the products are still being formed; the
// weight sits in shared memory.  A lane reads its row from TMEM twice (the
// mean square first; holding all 128 values measured slower).
template <bool GATED>
__device__ __forceinline__ void state_output_loop(uint8_t* smem, uint32_t tmem, const Maps& maps, const Params& p,
                                                  uint64_t* bars, volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = warp - 10;
  const int r = 32 * sub + lane;
  const uint32_t lane_off = static_cast<uint32_t>(64 + 32 * sub) << 16;
  uint8_t* st = smem + ST_OX + sub * 8192;  // [32 rows][128 v] bf16: two 64-value atoms of 4 KB
  int pos = 0;
  bool ok = true;
  StateWalk w{static_cast<int>(blockIdx.x) - p.R, 0, 0, 0};
  while (ok && w.next(p)) {
    const int h = w.ci % p.H;
    for (int j = 0; j < w.nc; ++j, ++pos) {
      const int b = pos & 1;
      const int64_t t0 = w.sb + static_cast<int64_t>(j) * C;
      const int L = static_cast<int>(w.se - t0 < C ? w.se - t0 : C);
      if constexpr (GATED) {
        // the previous tensor store out of the staging block must have read
        // it; then the chunk's 32 x 128 gate tile comes into it by TMA (rows
        // past the sequence end bring other rows or zeros: never stored)
        fence_proxy_async_smem();  // the last row-by-row pass read the block
        __syncwarp();
        if (lane == 0) {
          bulk_wait_read<0>();
          mbar_arrive_expect_tx(&bars[BS_G_FULL + sub], 8192);
          tma_load_2d(st, &maps.g, h * D, static_cast<int>(t0) + 32 * sub, &bars[BS_G_FULL + sub]);
          tma_load_2d(st + 4096, &maps.g, h * D + 64, static_cast<int>(t0) + 32 * sub, &bars[BS_G_FULL + sub]);
        }
        __syncwarp();
      }
      if (!mbar_wait_warp(&bars[BS_O_FULL + b], (pos >> 1) & 1, abort_flag)) {
        if constexpr (GATED) drain_tile(&bars[BS_G_FULL + sub], pos & 1);
        ok = false;
        break;
      }
      tc_fence_after();
      if constexpr (GATED) {
        // the row's mean square (one pass over TMEM), then the products again
        // (fp32 pairs: one packed instruction per two values)
        uint64_t ssa = 0, ssb = 0;
#pragma unroll 1
        for (int cb = 0; cb < 4; cb += 2) {
          float x[64];
          tmem_ld32(tmem + lane_off + TS_O + 128 * b + 32 * cb, *reinterpret_cast<float (*)[32]>(x));
          tmem_ld32(tmem + lane_off + TS_O + 128 * b + 32 * cb + 32, *reinterpret_cast<float (*)[32]>(x + 32));
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 64; u += 4) {
            const uint64_t xa = f2pack(x[u], x[u + 1]), xb = f2pack(x[u + 2], x[u + 3]);
            ssa = ffma2(xa, xa, ssa);
            ssb = ffma2(xb, xb, ssb);
          }
        }
        const float2 sa = f2unpack(ssa), sb = f2unpack(ssb);
        const float rinv = rsqrtf(((sa.x + sa.y) + (sb.x + sb.y)) * (1.f / D) + p.eps);
        // y = x (rinv / 2) (w + w tanh(g / 2)) = x / rms * w * sigmoid(g)
        const uint64_t hr2 = f2pack(0.5f * rinv, 0.5f * rinv), half2 = f2pack(0.5f, 0.5f);
        if (!mbar_wait_warp(&bars[BS_G_FULL + sub], pos & 1, abort_flag)) {
          drain_tile(&bars[BS_G_FULL + sub], pos & 1);
          ok = false;
          break;
        }
        const float* wsm = reinterpret_cast<const float*>(smem + ST_W);
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
          float x[32];
          tmem_ld32(tmem + lane_off + TS_O + 128 * b + 32 * cb, x);
          // the gate and weight of these 32 values, read while TMEM is
          uint4 gq[4];
          float4 wq[8];
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const int c0 = 32 * cb + 8 * j4;
            gq[j4] = lds128(st + (c0 >> 6) * 4096 + sw128(lane, (c0 & 63) >> 3));
            wq[2 * j4] = *reinterpret_cast<const float4*>(wsm + c0);
            wq[2 * j4 + 1] = *reinterpret_cast<const float4*>(wsm + c0 + 4);
          }
          tmem_wait_ld();
          // o / rms * w * sigmoid(g), written where the gate was
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const int c0 = 32 * cb + 8 * j4;
            const uint32_t g4[4] = {gq[j4].x, gq[j4].y, gq[j4].z, gq[j4].w};
            const float w8[8] = {wq[2 * j4].x, wq[2 * j4].y, wq[2 * j4].z, wq[2 * j4].w,
                                 wq[2 * j4 + 1].x, wq[2 * j4 + 1].y, wq[2 * j4 + 1].z, wq[2 * j4 + 1].w};
            uint32_t pk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 gv = bf2f(g4[u]);
              const float2 hg = f2unpack(fmul2(f2pack(gv.x, gv.y), half2));
              const uint64_t t2 = f2pack(tanh_approx(hg.x), tanh_approx(hg.y));
              const uint64_t w2 = f2pack(w8[2 * u], w8[2 * u + 1]);
              const float2 y = f2unpack(fmul2(fmul2(f2pack(x[8 * j4 + 2 * u], x[8 * j4 + 2 * u + 1]), hr2),
                                              ffma2(w2, t2, w2)));
              pk[u] = pack_bf16(y.x, y.y);
            }
            sts128(st + (c0 >> 6) * 4096 + sw128(lane, (c0 & 63) >> 3), make_uint4(pk[0], pk[1], pk[2], pk[3]));
          }
        }
        tc_fence_before();
        mbar_arrive(&bars[BS_O_FREE + b]);
      } else {
        // the previous tensor store out of the staging block must have read it
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll 1
        for (int cb = 0; cb < 4; ++cb) {
          float x[32];
          tmem_ld32(tmem + lane_off + TS_O + 128 * b + 32 * cb, x);
          tmem_wait_ld();
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const int vv = 32 * cb + 8 * j4;
            sts128(st + (vv >> 6) * 4096 + sw128(lane, (vv & 63) >> 3),
                   make_uint4(pack_bf16(x[8 * j4], x[8 * j4 + 1]), pack_bf16(x[8 * j4 + 2], x[8 * j4 + 3]),
                              pack_bf16(x[8 * j4 + 4], x[8 * j4 + 5]), pack_bf16(x[8 * j4 + 6], x[8 * j4 + 7])));
          }
        }
        tc_fence_before();
        mbar_arrive(&bars[BS_O_FREE + b]);
      }
      if (32 * sub + 32 <= L) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&maps.o, h * D, static_cast<int>(t0) + 32 * sub, st);
          tma_store_2d(&maps.o, h * D + 64, static_cast<int>(t0) + 32 * sub, st + 4096);
          bulk_commit();
        }
      } else {
        __syncwarp();
        if (r < L) {
#pragma unroll
          for (int c16 = 0; c16 < 16; ++c16)
            *reinterpret_cast<uint4*>(p.o + ((t0 + r) * p.H + h) * D + 8 * c16) =
                lds128(st + (c16 >> 3) * 4096 + sw128(lane, c16 & 7));
        }
        __syncwarp();
      }
    }
  }
  // tensor stores of O must be complete before the kernel ends
  if (lane == 0) bulk_wait_all();
}

// 8 warps; thread (q = warp & 3, hf = warp >> 2) owns value column v = 32 q + lane
// and channels [64 hf, 64 hf + 64) of S^T, in registers.
__device__ __forceinline__ void state_warps_loop(uint8_t* smem, uint32_t tmem, const Params& p, uint64_t* bars,
                                                 volatile int* abort_flag) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q = warp & 3, hf = warp >> 2;
  const int v = 32 * q + lane;
  const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
  const int i = blockIdx.x;
  float S[64];
  int pos = 0;
  bool ok = true;
  StateWalk w{i - p.R, 0, 0, 0};
  while (ok && w.next(p)) {
    const int n = w.ci / p.H, h = w.ci % p.H;
    bool rd, wr;
    const int row = state_row(p.st, n, &rd, &wr);
    const size_t sidx = (static_cast<size_t>(row < 0 ? 0 : row) * p.H + h) * D * D;
    if (rd) {
#pragma unroll
      for (int u = 0; u < 64; ++u) S[u] = p.st.S0[sidx + static_cast<size_t>(64 * hf + u) * D + v];
    } else {
#pragma unroll
      for (int u = 0; u < 64; ++u) S[u] = 0.f;
    }
    for (int j = 0; j < w.nc; ++j, ++pos) {
      const int s = pos & 1;
      const uint8_t* slot = smem + ST_A + s * SLOT_A;
      if (!mbar_wait_warp(&bars[BS_A_FULL + s], (pos >> 1) & 1, abort_flag)) { ok = false; break; }
      // S'^T = bf16(sc S^T) -> shared memory (A operand); S <- gamma_C S.  The
      // previous position's output product must have read the old S' first.
      {
        const float4* sc4 = reinterpret_cast<const float4*>(slot + R_VEC) + 16 * hf;
        uint32_t pk[32];
#pragma unroll
        for (int u4 = 0; u4 < 16; ++u4) {
          const float4 a = sc4[u4];
          pk[2 * u4] = pack_bf16(S[4 * u4] * a.x, S[4 * u4 + 1] * a.y);
          pk[2 * u4 + 1] = pack_bf16(S[4 * u4 + 2] * a.z, S[4 * u4 + 3] * a.w);
        }
        if (pos >= 1 && !mbar_wait_warp(&bars[BS_SP_FREE], (pos - 1) & 1, abort_flag)) { ok = false; break; }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          sts128(smem + ST_S + hf * 16384 + sw128(v, jj),
                 make_uint4(pk[4 * jj], pk[4 * jj + 1], pk[4 * jj + 2], pk[4 * jj + 3]));
        fence_proxy_async_smem();
        mbar_arrive(&bars[BS_S_READY]);
        const float4* gc4 = reinterpret_cast<const float4*>(slot + R_VEC) + 32 + 16 * hf;
#pragma unroll
        for (int u4 = 0; u4 < 16; ++u4) {
          const float4 gg = gc4[u4];
          S[4 * u4] *= gg.x;
          S[4 * u4 + 1] *= gg.y;
          S[4 * u4 + 2] *= gg.z;
          S[4 * u4 + 3] *= gg.w;
        }
      }
      // U^T -> bf16 shared memory (A operand)
      if (!mbar_wait_warp(&bars[BS_U_FULL], pos & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      {
        float x[32];
        tmem_ld32(tmem + lane_off + TS_U + 32 * hf, x);
        tmem_wait_ld();
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          uint32_t pk[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) pk[u] = pack_bf16(x[8 * j4 + 2 * u], x[8 * j4 + 2 * u + 1]);
          sts128(smem + ST_U + sw128(v, 4 * hf + j4), make_uint4(pk[0], pk[1], pk[2], pk[3]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[BS_U_READY]);
      // S += dS
      if (!mbar_wait_warp(&bars[BS_DS_FULL], pos & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      {
        float x[32];
        tmem_ld32(tmem + lane_off + TS_DS + 64 * hf, x);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) S[u] += x[u];
        tmem_ld32(tmem + lane_off + TS_DS + 64 * hf + 32, x);
        tmem_wait_ld();
#pragma unroll
        for (int u = 0; u < 32; ++u) S[32 + u] += x[u];
      }
      tc_fence_before();
    }
    if (!ok) break;
    if (wr) {
#pragma unroll
      for (int u = 0; u < 64; ++u) p.st.S_T[sidx + static_cast<size_t>(64 * hf + u) * D + v] = S[u];
    }
  }
}

// ===========================================================================
// the kernel
// ===========================================================================
template <typename TG, bool GATED, bool PROD>
__global__ void __launch_bounds__(NTHREADS, 1)
    kda_prefill_kernel(const __grid_constant__ Maps maps, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  using LY = TfLayout<TG>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool is_state = static_cast<int>(blockIdx.x) < p.R;
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars;
  uint32_t* tmem_slot;
  volatile int* abort_flag;
  int* s_maxlen = nullptr;  // transform CTAs: longest stream of any state CTA
  if (is_state) {
    bars = reinterpret_cast<uint64_t*>(smem + ST_BAR);
    tmem_slot = reinterpret_cast<uint32_t*>(smem + ST_BAR + 8 * BS_COUNT);
    abort_flag = reinterpret_cast<volatile int*>(smem + ST_BAR + 8 * BS_COUNT + 8);
  } else {
    bars = reinterpret_cast<uint64_t*>(smem + LY::MISC + LY::M_BAR);
    tmem_slot = reinterpret_cast<uint32_t*>(smem + LY::MISC + LY::NGROUP * LY::MISC_GROUP);
    abort_flag = reinterpret_cast<volatile int*>(smem + LY::MISC + LY::NGROUP * LY::MISC_GROUP + 8);
    s_maxlen = reinterpret_cast<int*>(smem + LY::MISC + LY::NGROUP * LY::MISC_GROUP + 16);
  }

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    if (!is_state) *s_maxlen = 0;
    if (is_state) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(&bars[BS_A_FULL + b], 1);
        mbar_init(&bars[BS_A_FREE + b], 1);
        mbar_init(&bars[BS_B_FULL + b], 1);
        mbar_init(&bars[BS_B_FREE + b], 1);
      }
      mbar_init(&bars[BS_S_READY], 256);
      mbar_init(&bars[BS_U_FULL], 1);
      mbar_init(&bars[BS_U_READY], 256);
      mbar_init(&bars[BS_DS_FULL], 1);
      mbar_init(&bars[BS_O_FULL + 0], 1);
      mbar_init(&bars[BS_O_FULL + 1], 1);
      mbar_init(&bars[BS_SP_FREE], 1);
      mbar_init(&bars[BS_O_FREE + 0], 64);
      mbar_init(&bars[BS_O_FREE + 1], 64);
      mbar_init(&bars[BS_FIN], 1);
      mbar_init(&bars[BS_G_FULL + 0], 1);
      mbar_init(&bars[BS_G_FULL + 1], 1);
    } else {
      for (int g = 0; g < LY::NGROUP; ++g) {
        uint64_t* gbars = reinterpret_cast<uint64_t*>(smem + LY::MISC + g * LY::MISC_GROUP + LY::M_BAR);
        for (int b = 0; b <= BT_WT_READ; ++b) mbar_init(&gbars[b], 1);
      }
    }
    fence_mbar_init();
  }
  if (!is_state) {
    // the cumsum operand [L; L], L[r][s] = (s <= r), bf16, K-major
    for (int e = threadIdx.x; e < 128 * 8; e += NTHREADS) {
      const int rr = e >> 3, jj = e & 7, r64 = rr & 63;
      uint32_t pk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = 8 * jj + 2 * u;
        pk[u] = pack_bf16(s <= r64 ? 1.f : 0.f, s + 1 <= r64 ? 1.f : 0.f);
      }
      sts128(smem + LY::L + sw128(rr, jj), make_uint4(pk[0], pk[1], pk[2], pk[3]));
    }
    fence_proxy_async_smem();
  }
  if constexpr (GATED) {
    if (is_state && threadIdx.x < D / 4)
      reinterpret_cast<float4*>(smem + ST_W)[threadIdx.x] = __ldg(reinterpret_cast<const float4*>(p.norm_w) + threadIdx.x);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (!is_state) {
    for (int i = threadIdx.x; i < p.R; i += NTHREADS) atomicMax(s_maxlen, stream_len(p, i));
    __syncthreads();
  }

  if (is_state) {
    if (warp < 8) {
      state_warps_loop(smem, tmem, p, bars, abort_flag);
    } else if (warp == 8) {
      if (lane == 0) state_load_loop(smem, maps, p, bars, abort_flag);
    } else if (warp == 9) {
      if (lane == 0) state_mma_loop(sbase, tmem, p, bars, abort_flag);
    } else {
      state_output_loop<GATED>(smem, tmem, maps, p, bars, abort_flag);
    }
  } else {
    const int g = (warp < 8) ? (warp >> 2) : ((warp - 8) & 1);
    if (g < LY::NGROUP) {
      Tf<TG, PROD> tf(smem, tmem, g);
      if (warp < 8) {
        tf.compute_loop(p, abort_flag);
      } else if (warp < 10) {
        tf.load_loop(maps, p, *s_maxlen, abort_flag);
      } else if (lane == 0) {
        tf.mma_loop(abort_flag);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) atomicExch(p.flags + F_ABORT, 1u);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace pipe
}  // namespace kda
