// kda_recurrent.cuh -- token-by-token KDA recurrence on CUDA cores, fp32.
//
// One CTA (256 threads) owns one (sequence, head) state S (DK x DV fp32) in
// registers for the whole run: thread (rg, cg) holds rows rg, rg+RP, ... and
// the four value columns 4cg..4cg+3, so a warp reads or writes whole 512-byte
// rows of S with 16-byte accesses.  Per token (the recurrence of the Kimi
// Linear articles' KDA layer, decay first, output from the updated state):
//     S~ = Diag(exp(log_alpha)) S
//     d  = beta (v - S~^T k)
//     S  = S~ + k d^T,      o = S^T q = S~^T q + (q.k) d
// The two column reductions (S~^T k, S~^T q) share one pass over S; partial
// sums meet in shared memory.
//
// Used for (a) kda_decode_step -- one token per (sequence, head), S read once
// and written once, a pure HBM stream -- and (b) kda_chunk_fwd whenever the
// tensor-core path does not apply (fp32 io, small head dims).
//
// PROD: the Kimi Linear layer's producer steps run here too: q and k arrive
// raw and are L2-normalised per token (the row sums of squares meet in
// shared memory), and the log-decay input holds the decay gate's projection
// f, log alpha = -exp(A_log[h]) * softplus(f + dt_bias[h][c]).  With a
// consumer (RecConsumer::gate set) the output epilogue runs on each token's
// o before it is stored: o / sqrt(mean(o^2) + eps) * w * sigmoid(g).  fp32
// io evaluates exp, log and the sigmoid with the accurate expf / log1pf (the
// 1e-4 tolerance of that path); bf16 io with the MUFU approximations.
#pragma once

#include "kda_ptx.cuh"
#include "kda_state_io.cuh"

namespace kda {

__device__ __forceinline__ float ld_f(const float* p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st_f(float* p, float x) { *p = x; }
__device__ __forceinline__ void st_f(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

constexpr int kRecThreads = 256;

// Producer parameters (PROD instantiations only).
struct RecProducer {
  const float* A_log = nullptr;    // [H]
  const float* dt_bias = nullptr;  // [H][DK]
};

// Output epilogue (gate == nullptr: none); gate has the io type, laid out like o.
struct RecConsumer {
  const void* gate = nullptr;
  const float* norm_w = nullptr;  // [DV]
  float eps = 0.f;
};

// softplus(x) = log(1 + e^x) and sigmoid(x): accurate for fp32 io, on the
// MUFU unit for bf16 io
template <typename TIO>
__device__ __forceinline__ float rec_softplus(float x) {
  if constexpr (sizeof(TIO) == 4) return x > 15.f ? x + log1pf(expf(-x)) : log1pf(expf(x));
  return x > 15.f ? x : 0.69314718f * lg2_approx(1.f + ex2_approx(x * 1.44269504f));
}
template <typename TIO>
__device__ __forceinline__ float rec_sigmoid(float x) {
  if constexpr (sizeof(TIO) == 4) return 1.f / (1.f + expf(-x));
  return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f);
}

template <int DK, int DV>
struct RecLayout {
  static constexpr int CG = DV / 4;                 // float4 column groups per row
  static constexpr int RP = kRecThreads / CG;       // rows covered per pass
  static constexpr int RPT = DK / RP;               // rows per thread
  static_assert(DK % RP == 0, "DK must be a multiple of the row pass");
};

template <int DK, int DV>
struct RecSmem {
  alignas(16) float delta[DV];  // read as float4
  float k[2][DK], qa[2][DK], a[2][DK], v[2][DV];
  float red_k[RecLayout<DK, DV>::RP][DV];
  float red_q[RecLayout<DK, DV>::RP][DV];
  float red_qk[RecLayout<DK, DV>::RP];
  float beta[2];
  float nk[2][DK / 32], nq[2][DK / 32];  // PROD: per-warp sums of k^2, q^2
  float no[DV / 32];                     // consumer: per-warp sums of o^2
};

// Runs tokens [t0, t1) of one (sequence, head).  Token t of head h lives at
// row (t * H + h) of the [*, H, d] inputs.  S_in / S_out may alias.
template <int DK, int DV, typename TIO, typename TG, bool kStream, bool PROD>
__device__ __forceinline__ void recurrent_run(int64_t t0, int64_t t1, int h, int H, const TIO* __restrict__ q,
                                              const TIO* __restrict__ k, const TIO* __restrict__ v,
                                              const TG* __restrict__ la, const TG* __restrict__ beta,
                                              const float* S_in, float* S_out, TIO* __restrict__ o,
                                              RecSmem<DK, DV>& sm, const RecProducer& pr, const RecConsumer& cs) {
  using L = RecLayout<DK, DV>;
  const int tid = threadIdx.x;
  const int cg = tid % L::CG;
  const int rg = tid / L::CG;

  float4 s[L::RPT];
  if (S_in) {
    const float4* src = reinterpret_cast<const float4*>(S_in);
#pragma unroll
    for (int i = 0; i < L::RPT; ++i) {
      const int r = rg + L::RP * i;
      s[i] = kStream ? __ldcs(src + r * L::CG + cg) : src[r * L::CG + cg];
    }
  } else {
#pragma unroll
    for (int i = 0; i < L::RPT; ++i) s[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  float nrate = 0.f, bias = 0.f;  // PROD: -exp(A_log[h]) and this thread's dt_bias[h][tid]
  if (PROD) {
    nrate = -expf(pr.A_log[h]);
    if (tid < DK) bias = pr.dt_bias[static_cast<int64_t>(h) * DK + tid];
  }
  int buf = 0;
  for (int64_t t = t0; t < t1; ++t, buf ^= 1) {
    const int64_t row = t * H + h;
    // stage this token's vectors (double-buffered across tokens)
    if (tid < DK) {
      float lav = ld_f(la + row * DK + tid);
      if (PROD) lav = nrate * rec_softplus<TIO>(lav + bias);
      sm.a[buf][tid] = __expf(lav);
      const float kv = ld_f(k + row * DK + tid), qv = ld_f(q + row * DK + tid);
      sm.k[buf][tid] = kv;
      sm.qa[buf][tid] = qv;
      if (PROD) {
        float ssk = kv * kv, ssq = qv * qv;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
          ssk += __shfl_xor_sync(0xffffffffu, ssk, m);
          ssq += __shfl_xor_sync(0xffffffffu, ssq, m);
        }
        if ((tid & 31) == 0) {
          sm.nk[buf][tid >> 5] = ssk;
          sm.nq[buf][tid >> 5] = ssq;
        }
      }
    }
    if (tid < DV) sm.v[buf][tid] = ld_f(v + row * DV + tid);
    if (tid == 0) sm.beta[buf] = ld_f(beta + row);
    __syncthreads();
    // PROD: 1/|k_t| and 1/|q_t| scale every use of k and q below
    float rk = 1.f, rq = 1.f;
    if (PROD) {
      float ssk = 0.f, ssq = 0.f;
#pragma unroll
      for (int w = 0; w < DK / 32; ++w) {
        ssk += sm.nk[buf][w];
        ssq += sm.nq[buf][w];
      }
      rk = rsqrtf(ssk + kQKNormEps);
      rq = rsqrtf(ssq + kQKNormEps);
    }

    // decay rows, then partial column sums of S~^T k and S~^T q
    float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f}, pqk = 0.f;
#pragma unroll
    for (int i = 0; i < L::RPT; ++i) {
      const int r = rg + L::RP * i;
      const float a = sm.a[buf][r], kr = sm.k[buf][r] * rk, qr = sm.qa[buf][r] * rq;
      s[i].x *= a;
      s[i].y *= a;
      s[i].z *= a;
      s[i].w *= a;
      pk[0] += kr * s[i].x; pk[1] += kr * s[i].y; pk[2] += kr * s[i].z; pk[3] += kr * s[i].w;
      pq[0] += qr * s[i].x; pq[1] += qr * s[i].y; pq[2] += qr * s[i].z; pq[3] += qr * s[i].w;
      pqk += kr * qr;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sm.red_k[rg][4 * cg + j] = pk[j];
      sm.red_q[rg][4 * cg + j] = pq[j];
    }
    if (cg == 0) sm.red_qk[rg] = pqk;
    __syncthreads();

    float ov = 0.f;
    if (tid < DV) {
      float ks = 0.f, qs = 0.f, qk = 0.f;
#pragma unroll
      for (int g = 0; g < L::RP; ++g) {
        ks += sm.red_k[g][tid];
        qs += sm.red_q[g][tid];
        qk += sm.red_qk[g];
      }
      const float d = sm.beta[buf] * (sm.v[buf][tid] - ks);
      sm.delta[tid] = d;
      ov = qs + qk * d;
      if (cs.gate) {
        float so = ov * ov;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) so += __shfl_xor_sync(0xffffffffu, so, m);
        if ((tid & 31) == 0) sm.no[tid >> 5] = so;
      } else {
        st_f(o + row * DV + tid, ov);
      }
    }
    __syncthreads();
    if (cs.gate && tid < DV) {
      float so = 0.f;
#pragma unroll
      for (int w = 0; w < DV / 32; ++w) so += sm.no[w];
      const float g = ld_f(static_cast<const TIO*>(cs.gate) + row * DV + tid);
      st_f(o + row * DV + tid, ov * rsqrtf(so * (1.f / DV) + cs.eps) * cs.norm_w[tid] * rec_sigmoid<TIO>(g));
    }

    const float4 d4 = reinterpret_cast<const float4*>(sm.delta)[cg];
#pragma unroll
    for (int i = 0; i < L::RPT; ++i) {
      const float kr = sm.k[buf][rg + L::RP * i] * rk;
      s[i].x += kr * d4.x;
      s[i].y += kr * d4.y;
      s[i].z += kr * d4.z;
      s[i].w += kr * d4.w;
    }
  }

  if (S_out) {
    float4* dst = reinterpret_cast<float4*>(S_out);
#pragma unroll
    for (int i = 0; i < L::RPT; ++i) {
      const int r = rg + L::RP * i;
      if (kStream)
        __stcs(dst + r * L::CG + cg, s[i]);
      else
        dst[r * L::CG + cg] = s[i];
    }
  }
}

// Decode: blockIdx.x = n * H + h; token n of the [N, H, d] inputs.  The state
// of sequence n is row n of S, or pool slot slots[n] when slots is given; a
// negative slot has no cached state: the token runs from a zero state and the
// new state is dropped.
template <int DK, int DV, typename TIO, typename TG, bool PROD>
__global__ void __launch_bounds__(kRecThreads, 2)
    kda_decode_kernel(int H, const TIO* __restrict__ q, const TIO* __restrict__ k, const TIO* __restrict__ v,
                      const TG* __restrict__ la, const TG* __restrict__ beta, float* S, TIO* __restrict__ o,
                      const int32_t* __restrict__ slots, int num_slots, RecProducer pr, RecConsumer cs) {
  __shared__ __align__(16) RecSmem<DK, DV> sm;
  const int nh = blockIdx.x;
  const int n = nh / H, h = nh % H;
  StateIO io;
  io.S0 = S;
  io.S_T = S;
  io.slots = slots;
  io.num_slots = num_slots;
  bool rd, wr;
  const int row = state_row(io, n, &rd, &wr);
  float* Snh = S + (static_cast<int64_t>(row < 0 ? 0 : row) * H + h) * DK * DV;
  recurrent_run<DK, DV, TIO, TG, true, PROD>(n, n + 1, h, H, q, k, v, la, beta, rd ? Snh : nullptr,
                                             wr ? Snh : nullptr, o, sm, pr, cs);
}

// Prefill on CUDA cores: blockIdx.x = h, blockIdx.y = sequence n.
template <int DK, int DV, typename TIO, typename TG, bool PROD>
__global__ void __launch_bounds__(kRecThreads, 2)
    kda_recurrent_fwd_kernel(int H, int T, const int32_t* __restrict__ cu_seqlens, const TIO* __restrict__ q,
                             const TIO* __restrict__ k, const TIO* __restrict__ v, const TG* __restrict__ la,
                             const TG* __restrict__ beta, StateIO io, TIO* __restrict__ o, RecProducer pr,
                             RecConsumer cs) {
  __shared__ __align__(16) RecSmem<DK, DV> sm;
  const int h = blockIdx.x, n = blockIdx.y;
  int64_t t0, t1;
  if (cu_seqlens) {
    t0 = cu_seqlens[n];
    t1 = cu_seqlens[n + 1];
  } else {
    t0 = static_cast<int64_t>(n) * T;
    t1 = t0 + T;
  }
  bool rd, wr;
  const int row = state_row(io, n, &rd, &wr);
  const int64_t off = (static_cast<int64_t>(row < 0 ? 0 : row) * H + h) * DK * DV;
  recurrent_run<DK, DV, TIO, TG, false, PROD>(t0, t1, h, H, q, k, v, la, beta, rd ? io.S0 + off : nullptr,
                                              wr ? io.S_T + off : nullptr, o, sm, pr, cs);
}

}  // namespace kda
