// kda_api.cu -- host side of libkda.so: argument validation, path selection
// and kernel launches behind the extern "C" entry points of include/kda.h.
// Every check runs on the host before anything is launched; no entry point
// allocates device memory, aborts or prints.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <vector>

#include "kda.h"
#include "kda_prefill.cuh"
#include "kda_recurrent.cuh"
#include "kda_tma.h"

namespace {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline bool aligned16(const void* p) { return aligned(p, 16); }
inline uintptr_t gate_size(const kda_shape& s) { return s.gate_dtype == KDA_BF16 ? 2 : 4; }
// Alignment each kernel relies on: 16 bytes for fp32 states (float4) and the
// workspace, 4 bytes for token tensors (bf16 pairs), element size for beta.
inline bool token_ptrs_aligned(const kda_shape& s, const void* q, const void* k, const void* v, const void* la,
                               const void* beta, const void* o) {
  return aligned(q, 4) && aligned(k, 4) && aligned(v, 4) && aligned(la, 4) && aligned(o, 4) &&
         aligned(beta, gate_size(s));
}
inline bool dtype_ok(int32_t d) { return d == KDA_F32 || d == KDA_BF16; }
inline bool dim_ok(int32_t d) { return d == 64 || d == 128; }

// Tensor-core chunk path: bf16 io and dk = dv = 128 (chunk C = 64), unless
// KDA_FLAG_PATH_RECURRENT asks for the token-by-token CUDA-core recurrence.
inline bool use_tc(const kda_shape& s) {
  return s.io_dtype == KDA_BF16 && s.dk == 128 && s.dv == 128 && (s.flags & KDA_FLAG_PATH_RECURRENT) == 0u;
}
constexpr uint32_t kKnownFlags = KDA_FLAG_VALIDATE_CU_SEQLENS | KDA_FLAG_PATH_RECURRENT | KDA_FLAG_GATE_FUSED |
                                  KDA_FLAG_GATE_SEPARATE | KDA_FLAG_STATE_CTAS(0xFF) | KDA_FLAG_GRID_CTAS(0xFF);

// Number of sequences N and the packed token total.
inline void seq_counts(const kda_shape& s, const int32_t* cu, int64_t* N, int64_t* Ttot) {
  if (cu) {
    *N = s.n_seqs;
    *Ttot = s.T;
  } else {
    *N = s.B;
    *Ttot = static_cast<int64_t>(s.B) * s.T;
  }
}

kda_status check_common(const kda_shape* sp) {
  if (!sp) return KDA_ERR_NULL;
  const kda_shape& s = *sp;
  if (!dtype_ok(s.io_dtype) || !dtype_ok(s.gate_dtype)) return KDA_ERR_DTYPE;
  if (s.B <= 0 || s.T < 0 || s.H <= 0) return KDA_ERR_SHAPE;
  if (!dim_ok(s.dk) || !dim_ok(s.dv)) return KDA_ERR_UNSUPPORTED;
  if ((s.flags & ~kKnownFlags) != 0u) return KDA_ERR_ARGUMENT;
  if ((s.flags & KDA_FLAG_GATE_FUSED) && (s.flags & KDA_FLAG_GATE_SEPARATE)) return KDA_ERR_ARGUMENT;
  return KDA_OK;
}

kda_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

template <int DK, int DV, typename TIO, typename TG>
kda_status launch_recurrent_fwd(const kda_shape& s, int64_t N, const void* q, const void* k, const void* v,
                                const void* la, const void* beta, const kda::StateIO& io, const int32_t* cu,
                                void* o, cudaStream_t st, const kda::RecProducer& pr, const kda::RecConsumer& cs) {
  dim3 grid(s.H, static_cast<unsigned>(N));
  auto* kern = pr.A_log ? kda::kda_recurrent_fwd_kernel<DK, DV, TIO, TG, true>
                        : kda::kda_recurrent_fwd_kernel<DK, DV, TIO, TG, false>;
  kern<<<grid, kda::kRecThreads, 0, st>>>(s.H, s.T, cu, static_cast<const TIO*>(q), static_cast<const TIO*>(k),
                                          static_cast<const TIO*>(v), static_cast<const TG*>(la),
                                          static_cast<const TG*>(beta), io, static_cast<TIO*>(o), pr, cs);
  return launch_status();
}

template <typename TIO, typename TG>
kda_status dispatch_recurrent_fwd(const kda_shape& s, int64_t N, const void* q, const void* k, const void* v,
                                  const void* la, const void* beta, const kda::StateIO& io, const int32_t* cu,
                                  void* o, cudaStream_t st, const kda::RecProducer& pr,
                                  const kda::RecConsumer& cs) {
  if (s.dk == 128 && s.dv == 128)
    return launch_recurrent_fwd<128, 128, TIO, TG>(s, N, q, k, v, la, beta, io, cu, o, st, pr, cs);
  if (s.dk == 64 && s.dv == 64)
    return launch_recurrent_fwd<64, 64, TIO, TG>(s, N, q, k, v, la, beta, io, cu, o, st, pr, cs);
  if (s.dk == 128 && s.dv == 64)
    return launch_recurrent_fwd<128, 64, TIO, TG>(s, N, q, k, v, la, beta, io, cu, o, st, pr, cs);
  return launch_recurrent_fwd<64, 128, TIO, TG>(s, N, q, k, v, la, beta, io, cu, o, st, pr, cs);
}

template <int DK, int DV, typename TIO, typename TG>
kda_status launch_decode(const kda_shape& s, const void* q, const void* k, const void* v, const void* la,
                         const void* beta, float* S, const int32_t* slots, int num_slots, void* o,
                         cudaStream_t st, const kda::RecProducer& pr, const kda::RecConsumer& cs) {
  const unsigned blocks = static_cast<unsigned>(s.B) * static_cast<unsigned>(s.H);
  auto* kern = pr.A_log ? kda::kda_decode_kernel<DK, DV, TIO, TG, true> : kda::kda_decode_kernel<DK, DV, TIO, TG, false>;
  kern<<<blocks, kda::kRecThreads, 0, st>>>(s.H, static_cast<const TIO*>(q), static_cast<const TIO*>(k),
                                            static_cast<const TIO*>(v), static_cast<const TG*>(la),
                                            static_cast<const TG*>(beta), S, static_cast<TIO*>(o), slots, num_slots,
                                            pr, cs);
  return launch_status();
}

template <typename TIO, typename TG>
kda_status dispatch_decode(const kda_shape& s, const void* q, const void* k, const void* v, const void* la,
                           const void* beta, float* S, const int32_t* slots, int num_slots, void* o,
                           cudaStream_t st, const kda::RecProducer& pr, const kda::RecConsumer& cs) {
  if (s.dk == 128 && s.dv == 128)
    return launch_decode<128, 128, TIO, TG>(s, q, k, v, la, beta, S, slots, num_slots, o, st, pr, cs);
  if (s.dk == 64 && s.dv == 64)
    return launch_decode<64, 64, TIO, TG>(s, q, k, v, la, beta, S, slots, num_slots, o, st, pr, cs);
  if (s.dk == 128 && s.dv == 64)
    return launch_decode<128, 64, TIO, TG>(s, q, k, v, la, beta, S, slots, num_slots, o, st, pr, cs);
  return launch_decode<64, 128, TIO, TG>(s, q, k, v, la, beta, S, slots, num_slots, o, st, pr, cs);
}

// Opt-in to large dynamic shared memory.  Set on every launch: the call is
// a cheap host-side attribute update, and caching it per device would go
// stale if the caller resets the device (the attribute dies with the context).
template <typename F>
bool ensure_smem(F* kernel, uint32_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) ==
         cudaSuccess;
}

// ---------------------------------------------------------------------------
// Pipelined tensor-core prefill (kda_prefill.cuh)
// ---------------------------------------------------------------------------
int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Optional output epilogue of the tensor-core prefill (gate == nullptr: none).
struct Epilogue {
  const void* gate = nullptr;
  const float* norm_w = nullptr;
  float eps = 0.f;
};

// Optional producer steps of the tensor-core prefill (A_log == nullptr: none):
// q, k are L2-normalised in the kernel and log_alpha carries the decay gate's
// projection f, log alpha = -exp(A_log[h]) * softplus(f + dt_bias[h][c]).
struct Producer {
  const float* A_log = nullptr;
  const float* dt_bias = nullptr;
};

struct PrefillPlan {
  int R = 0;             // state CTAs
  bool fuse_gate = false;  // output epilogue in the state CTAs (they have time to spare)
  int grid = 0;          // all CTAs (one per SM)
  size_t flag_bytes = 0; // zeroed before each launch
  size_t ring_off = 0;
  size_t ring_unit = 0;  // bytes per ring slot of every state CTA
  size_t bytes = 0;      // preferred workspace: the deepest ring
  size_t min_bytes = 0;  // smallest usable workspace: a 2-slot ring
  // ring depth a workspace of ws_bytes allows (0 if too small)
  int nring(size_t ws_bytes) const {
    if (ws_bytes < min_bytes) return 0;
    const size_t d = (ws_bytes - ring_off) / ring_unit;
    return static_cast<int>(d < static_cast<size_t>(kda::pipe::MAX_RING) ? d : kda::pipe::MAX_RING);
  }
};

// Splits the SMs between state CTAs (one serial chain of chunks each) and
// transform CTAs (parallel per-chunk work).  With `chains` (sequence, head)
// pairs and a grid of G CTAs, R state CTAs take ceil(chains / R) chains each,
// and the G - R transform CTAs share all chunks; a transform CTA needs about
// kTransformCost times as long per chunk as a state CTA spends on one chunk
// of its chain.  R minimises the larger of the two times.
constexpr double kTransformCost = 2.0;
// The fused output epilogue keeps the state CTAs' two output warps busy for
// about as long as a state CTA spends on a chunk, so it is free only where
// the transform CTAs bound the call: it is fused where the transform side's
// time exceeds the state side's by kFuseMargin, else it runs as a separate
// pass over o.  (Measured on B200: fused wins on the 4 x 4096 and the
// 8-sequence varlen prefills, the separate pass on one 128K-token sequence.)
constexpr double kFuseMargin = 1.05;
constexpr size_t kRingL2Bytes = 48u << 20;
constexpr int kMinPreferredRing = 4;

PrefillPlan plan_prefill(const kda_shape& s, int64_t N, int nsm) {
  PrefillPlan pl;
  const int64_t chains = N * s.H;
  int grid = nsm;
  const int grid_req = static_cast<int>((s.flags >> 16) & 0xFFu);
  if (grid_req > 0 && grid_req < grid) grid = grid_req;
  if (grid < 2 || chains <= 0) return pl;
  const int rmax = static_cast<int>(chains < grid - 1 ? chains : grid - 1);
  int R = static_cast<int>((s.flags >> 8) & 0xFFu);
  if (R > 0) {
    R = R < rmax ? R : rmax;
  } else {
    double best = 1e300;
    for (int r = 1; r <= rmax; ++r) {
      const double t_state = static_cast<double>((chains + r - 1) / r);
      const double t_tf = static_cast<double>(chains) * kTransformCost / (grid - r);
      const double t = t_state > t_tf ? t_state : t_tf;
      if (t < best - 1e-9) {
        best = t;
        R = r;
      }
    }
  }
  pl.R = R;
  pl.grid = grid;
  {
    const double t_state = static_cast<double>((chains + R - 1) / R);
    const double t_tf = static_cast<double>(chains) * kTransformCost / (grid - R);
    pl.fuse_gate = t_state * kFuseMargin <= t_tf;
  }
  pl.flag_bytes = kda::pipe::flag_words(R) * sizeof(uint32_t);
  pl.ring_off = (pl.flag_bytes + 1023) & ~static_cast<size_t>(1023);
  pl.ring_unit = static_cast<size_t>(R) * kda::pipe::SLOT;
  // preferred depth: as deep as kRingL2Bytes of ring allows (the ring should
  // stay in L2 next to the streaming inputs: a deeper ring is written back to
  // HBM), at least kMinPreferredRing slots
  int depth = static_cast<int>(kRingL2Bytes / pl.ring_unit);
  depth = depth < kMinPreferredRing ? kMinPreferredRing : depth;
  depth = depth > kda::pipe::MAX_RING ? kda::pipe::MAX_RING : depth;
  pl.bytes = pl.ring_off + pl.ring_unit * depth;
  pl.min_bytes = pl.ring_off + pl.ring_unit * 2;
  return pl;
}

// With an epilogue, *fused says whether the kernel applied it (else the caller
// runs the separate pass).
template <typename TG, bool PROD>
kda_status launch_prefill(const kda_shape& s, int64_t N, int64_t Ttot, const void* q, const void* k, const void* v,
                          const void* la, const void* beta, const kda::StateIO& io, const Epilogue& ep_req,
                          const Producer& pr, const int32_t* cu, void* o,
                          void* ws, size_t ws_bytes, cudaStream_t st, bool* fused) {
  namespace P = kda::pipe;
  const PrefillPlan pl = plan_prefill(s, N, device_sm_count());
  const bool fuse = ep_req.gate != nullptr && ((s.flags & KDA_FLAG_GATE_FUSED) != 0u ||
                                               ((s.flags & KDA_FLAG_GATE_SEPARATE) == 0u && pl.fuse_gate));
  const Epilogue ep = fuse ? ep_req : Epilogue{};
  *fused = fuse;
  if (pl.R <= 0) return KDA_ERR_CUDA;
  const int nring = pl.nring(ws_bytes);
  if (!ws || nring < 2) return KDA_ERR_WORKSPACE;
  // the work-item counter is 32-bit: R * (chunks of the longest stream) must fit
  if (static_cast<double>(pl.R) * (static_cast<double>(Ttot) / P::C + static_cast<double>(N)) > 2.0e9)
    return KDA_ERR_SHAPE;
  P::Maps maps = {};
  const uint64_t cols = static_cast<uint64_t>(s.H) * P::D;
  const uint64_t rows = static_cast<uint64_t>(Ttot);
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  bool ok = kda::make_tma_2d(&maps.q, q, bf, 2, cols, rows, cols * 2, 64, 64) &&
            kda::make_tma_2d(&maps.k, k, bf, 2, cols, rows, cols * 2, 64, 64) &&
            kda::make_tma_2d(&maps.v, v, bf, 2, cols, rows, cols * 2, 64, 64) &&
            kda::make_tma_2d(&maps.o, o, bf, 2, cols, rows, cols * 2, 64, 32);
  if (ep.gate) ok = ok && kda::make_tma_2d(&maps.g, ep.gate, bf, 2, cols, rows, cols * 2, 64, 32);
  if (sizeof(TG) == 2)
    ok = ok && kda::make_tma_2d(&maps.la, la, bf, 2, cols, rows, cols * 2, 64, 64);
  else
    ok = ok && kda::make_tma_2d(&maps.la, la, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, cols, rows, cols * 4, 32, 64);
  if (!ok) return kda::tma_encode_fn() ? KDA_ERR_ALIGN : KDA_ERR_CUDA;
  P::Params prm;
  prm.T = s.T;
  prm.H = s.H;
  prm.N = static_cast<int>(N);
  prm.R = pl.R;
  prm.nring = nring;
  prm.cu = cu;
  prm.beta = beta;
  prm.st = io;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.A_log = pr.A_log;
  prm.dt_bias = pr.dt_bias;
  prm.gate = static_cast<const __nv_bfloat16*>(ep.gate);
  prm.norm_w = ep.norm_w;
  prm.eps = ep.eps;
  prm.flags = static_cast<uint32_t*>(ws);
  prm.ring = static_cast<uint8_t*>(ws) + pl.ring_off;
  auto* kern = ep.gate ? P::kda_prefill_kernel<TG, true, PROD> : P::kda_prefill_kernel<TG, false, PROD>;
  const uint32_t smem = P::ST_BYTES > P::TfLayout<TG>::BYTES ? P::ST_BYTES : P::TfLayout<TG>::BYTES;
  if (!ensure_smem(kern, smem)) return KDA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, pl.flag_bytes, st) != cudaSuccess) return KDA_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
  cfg.blockDim = dim3(P::NTHREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, maps, prm) != cudaSuccess) {
    (void)cudaGetLastError();
    return KDA_ERR_CUDA;
  }
  return KDA_OK;
}

// The output epilogue as its own pass over o (kda_epilogue.cuh).
template <typename TO>
kda_status launch_output_gate(TO* o, const void* gate, const float* w, float eps, int64_t rows, int dv,
                              cudaStream_t st) {
  namespace E = kda::epi;
  const int rows_per_block = E::kThreads / (dv / 8);
  const int64_t want = (rows + 2 * rows_per_block - 1) / (2 * rows_per_block);
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
  const unsigned blocks = static_cast<unsigned>(want < cap ? (want > 0 ? want : 1) : (cap > 0 ? cap : 1));
  const TO* g = static_cast<const TO*>(gate);
  if (dv == 128)
    E::kda_output_gate_kernel<TO, 128><<<blocks, E::kThreads, 0, st>>>(o, g, w, eps, rows);
  else
    E::kda_output_gate_kernel<TO, 64><<<blocks, E::kThreads, 0, st>>>(o, g, w, eps, rows);
  return launch_status();
}

kda_status validate_cu_host(const int32_t* cu, int64_t N, int64_t Ttot, cudaStream_t st) {
  std::vector<int32_t> h(static_cast<size_t>(N) + 1);
  if (cudaMemcpyAsync(h.data(), cu, h.size() * sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return KDA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return KDA_ERR_CUDA;
  if (h[0] != 0 || h[N] != Ttot) return KDA_ERR_ARGUMENT;
  for (int64_t i = 0; i < N; ++i)
    if (h[i + 1] < h[i]) return KDA_ERR_ARGUMENT;
  return KDA_OK;
}

}  // namespace

extern "C" {

size_t kda_chunk_fwd_workspace_size(const kda_shape* sp) {
  if (check_common(sp) != KDA_OK) return 0;
  const kda_shape& s = *sp;
  if (!use_tc(s)) return 0;
  const bool packed = s.n_seqs > 0 && s.B == 1;
  const int64_t N = packed ? s.n_seqs : s.B;
  return plan_prefill(s, N, device_sm_count()).bytes;
}

kda_status kda_prefill_plan(const kda_shape* sp, int32_t num_sms, kda_prefill_plan_info* out) {
  if (!out) return KDA_ERR_NULL;
  const kda_status e = check_common(sp);
  if (e != KDA_OK) return e;
  const kda_shape& s = *sp;
  if (!use_tc(s)) return KDA_ERR_UNSUPPORTED;
  if (num_sms <= 0) num_sms = device_sm_count();
  if (num_sms <= 0) return KDA_ERR_CUDA;
  const bool packed = s.n_seqs > 0 && s.B == 1;
  const int64_t N = packed ? s.n_seqs : s.B;
  const PrefillPlan pl = plan_prefill(s, N, num_sms);
  if (pl.R <= 0) return KDA_ERR_SHAPE;
  out->state_ctas = pl.R;
  out->grid_ctas = pl.grid;
  out->ring_depth = pl.nring(pl.bytes);
  out->fuse_output_gate = (s.flags & KDA_FLAG_GATE_FUSED) != 0u     ? 1
                          : (s.flags & KDA_FLAG_GATE_SEPARATE) != 0u ? 0
                                                                     : (pl.fuse_gate ? 1 : 0);
  out->workspace_bytes = pl.bytes;
  out->min_workspace_bytes = pl.min_bytes;
  return KDA_OK;
}

}  // extern "C"

namespace {
// Smallest workspace kda_chunk_fwd accepts: the pipelined path runs with any
// ring depth from 2 to 16 slots per state CTA.
size_t kda_chunk_fwd_min_workspace(const kda_shape* sp) {
  if (check_common(sp) != KDA_OK) return 0;
  const kda_shape& s = *sp;
  if (!use_tc(s)) return 0;
  const bool packed = s.n_seqs > 0 && s.B == 1;
  const int64_t N = packed ? s.n_seqs : s.B;
  return plan_prefill(s, N, device_sm_count()).min_bytes;
}

// Shared body of kda_chunk_fwd and kda_chunk_fwd_slots; `io` says where the
// states live (dense rows or pool slots).
kda_status chunk_fwd(const kda_shape* sp, const void* q, const void* k, const void* v, const void* log_alpha,
                     const void* beta, const kda::StateIO& io, const Epilogue& ep, const Producer& pr,
                     const int32_t* cu_seqlens,
                     void* o, void* workspace,
                     size_t workspace_bytes, void* stream) {
  kda_status e = check_common(sp);
  if (e != KDA_OK) return e;
  const kda_shape& s = *sp;
  if (s.chunk != 64) return KDA_ERR_UNSUPPORTED;
  if (cu_seqlens && (s.B != 1 || s.n_seqs <= 0)) return KDA_ERR_SHAPE;
  int64_t N, Ttot;
  seq_counts(s, cu_seqlens, &N, &Ttot);
  const bool any_tokens = Ttot > 0;
  if (any_tokens && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_NULL;
  if (!token_ptrs_aligned(s, q, k, v, log_alpha, beta, o) || !aligned16(io.S0) || !aligned16(io.S_T) ||
      !aligned(cu_seqlens, 4))
    return KDA_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cu_seqlens && (s.flags & KDA_FLAG_VALIDATE_CU_SEQLENS)) {
    e = validate_cu_host(cu_seqlens, N, Ttot, st);
    if (e != KDA_OK) return e;
  }
  if (N == 0) return KDA_OK;

  if (ep.gate && Ttot > 0 && (!aligned16(o) || !aligned16(ep.gate))) return KDA_ERR_ALIGN;
  bool fused = false;
  if (pr.A_log && use_tc(s) && s.gate_dtype != KDA_BF16) return KDA_ERR_UNSUPPORTED;
  kda::RecProducer rp;
  rp.A_log = pr.A_log;
  rp.dt_bias = pr.dt_bias;
  kda::RecConsumer rc;  // the CUDA-core kernels apply the output epilogue themselves
  rc.gate = ep.gate;
  rc.norm_w = ep.norm_w;
  rc.eps = ep.eps;
  if (pr.A_log && use_tc(s) && Ttot > 0) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(log_alpha) || !aligned16(o) ||
        !aligned16(pr.dt_bias))
      return KDA_ERR_ALIGN;
    e = launch_prefill<__nv_bfloat16, true>(s, N, Ttot, q, k, v, log_alpha, beta, io, ep, pr, cu_seqlens, o,
                                            workspace, workspace_bytes, st, &fused);
  } else if (use_tc(s) && Ttot > 0) {
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(log_alpha) || !aligned16(o))
      return KDA_ERR_ALIGN;
    if (s.gate_dtype == KDA_BF16)
      e = launch_prefill<__nv_bfloat16, false>(s, N, Ttot, q, k, v, log_alpha, beta, io, ep, pr, cu_seqlens, o,
                                               workspace, workspace_bytes, st, &fused);
    else
      e = launch_prefill<float, false>(s, N, Ttot, q, k, v, log_alpha, beta, io, ep, pr, cu_seqlens, o, workspace,
                                       workspace_bytes, st, &fused);
  } else if (s.io_dtype == KDA_F32) {
    fused = ep.gate != nullptr;
    if (s.gate_dtype == KDA_F32)
      e = dispatch_recurrent_fwd<float, float>(s, N, q, k, v, log_alpha, beta, io, cu_seqlens, o, st, rp, rc);
    else
      e = dispatch_recurrent_fwd<float, __nv_bfloat16>(s, N, q, k, v, log_alpha, beta, io, cu_seqlens, o, st,
                                                           rp, rc);
  } else if (s.gate_dtype == KDA_F32) {
    fused = ep.gate != nullptr;
    e = dispatch_recurrent_fwd<__nv_bfloat16, float>(s, N, q, k, v, log_alpha, beta, io, cu_seqlens, o, st, rp, rc);
  } else {
    fused = ep.gate != nullptr;
    e = dispatch_recurrent_fwd<__nv_bfloat16, __nv_bfloat16>(s, N, q, k, v, log_alpha, beta, io, cu_seqlens, o,
                                                             st, rp, rc);
  }
  if (e != KDA_OK || !ep.gate || fused || Ttot == 0) return e;
  const int64_t rows = Ttot * s.H;
  if (s.io_dtype == KDA_F32)
    return launch_output_gate<float>(static_cast<float*>(o), ep.gate, ep.norm_w, ep.eps, rows, s.dv, st);
  return launch_output_gate<__nv_bfloat16>(static_cast<__nv_bfloat16*>(o), ep.gate, ep.norm_w, ep.eps, rows, s.dv,
                                           st);
}

// Shared body of kda_decode_step and kda_decode_step_slots.
kda_status decode_step(const kda_shape* sp, const void* q, const void* k, const void* v, const void* log_alpha,
                       const void* beta, float* S, const int32_t* slots, int num_slots, void* o, void* stream,
                       const kda::RecProducer& pr = kda::RecProducer{}, const Epilogue& ep = Epilogue{}) {
  kda_status e = check_common(sp);
  if (e != KDA_OK) return e;
  const kda_shape& s = *sp;
  if (s.T != 1) return KDA_ERR_SHAPE;
  if (!q || !k || !v || !log_alpha || !beta || !S || !o) return KDA_ERR_NULL;
  if (!token_ptrs_aligned(s, q, k, v, log_alpha, beta, o) || !aligned16(S) || !aligned(slots, 4))
    return KDA_ERR_ALIGN;
  if (static_cast<int64_t>(s.B) * s.H > 0x7fffffffLL) return KDA_ERR_SHAPE;
  if (ep.gate && (!aligned(ep.gate, s.io_dtype == KDA_F32 ? 4 : 2) || !aligned(ep.norm_w, 4))) return KDA_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  kda::RecConsumer cs;  // the output epilogue, in the kernel
  cs.gate = ep.gate;
  cs.norm_w = ep.norm_w;
  cs.eps = ep.eps;
  if (s.io_dtype == KDA_F32) {
    if (s.gate_dtype == KDA_F32)
      return dispatch_decode<float, float>(s, q, k, v, log_alpha, beta, S, slots, num_slots, o, st, pr, cs);
    return dispatch_decode<float, __nv_bfloat16>(s, q, k, v, log_alpha, beta, S, slots, num_slots, o, st, pr, cs);
  }
  if (s.gate_dtype == KDA_F32)
    return dispatch_decode<__nv_bfloat16, float>(s, q, k, v, log_alpha, beta, S, slots, num_slots, o, st, pr, cs);
  return dispatch_decode<__nv_bfloat16, __nv_bfloat16>(s, q, k, v, log_alpha, beta, S, slots, num_slots, o, st, pr,
                                                       cs);
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd(const kda_shape* sp, const void* q, const void* k, const void* v, const void* log_alpha,
                         const void* beta, const float* S0, const int32_t* cu_seqlens, void* o, float* S_T,
                         void* workspace, size_t workspace_bytes, void* stream) {
  kda::StateIO io;
  io.S0 = S0;
  io.S_T = S_T;
  return chunk_fwd(sp, q, k, v, log_alpha, beta, io, Epilogue{}, Producer{}, cu_seqlens, o, workspace,
                   workspace_bytes, stream);
}

kda_status kda_chunk_fwd_slots(const kda_shape* sp, const void* q, const void* k, const void* v,
                               const void* log_alpha, const void* beta, float* state_pool, int32_t num_slots,
                               const int32_t* state_slots, const uint8_t* has_initial_state,
                               const int32_t* cu_seqlens, void* o, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (!state_pool || !state_slots) return KDA_ERR_NULL;
  if (num_slots <= 0) return KDA_ERR_SHAPE;
  if (!aligned(state_slots, 4)) return KDA_ERR_ALIGN;
  kda::StateIO io;
  io.S0 = state_pool;
  io.S_T = state_pool;
  io.slots = state_slots;
  io.has_init = has_initial_state;
  io.num_slots = num_slots;
  return chunk_fwd(sp, q, k, v, log_alpha, beta, io, Epilogue{}, Producer{}, cu_seqlens, o, workspace,
                   workspace_bytes, stream);
}

kda_status kda_chunk_fwd_gated(const kda_shape* sp, const void* q, const void* k, const void* v,
                               const void* log_alpha, const void* beta, const float* S0, const int32_t* cu_seqlens,
                               const void* out_gate, const float* norm_weight, float eps, void* o, float* S_T,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (!sp) return KDA_ERR_NULL;
  if (!out_gate || !norm_weight) return KDA_ERR_NULL;
  if (!(eps >= 0.f) || !(eps < 3.0e38f)) return KDA_ERR_ARGUMENT;
  if (!aligned16(out_gate) || !aligned16(norm_weight)) return KDA_ERR_ALIGN;
  kda::StateIO io;
  io.S0 = S0;
  io.S_T = S_T;
  Epilogue ep;
  ep.gate = out_gate;
  ep.norm_w = norm_weight;
  ep.eps = eps;
  return chunk_fwd(sp, q, k, v, log_alpha, beta, io, ep, Producer{}, cu_seqlens, o, workspace, workspace_bytes,
                   stream);
}

kda_status kda_chunk_fwd_layer(const kda_shape* sp, const void* q, const void* k, const void* v, const void* gate_f,
                               const float* A_log, const float* dt_bias, const void* beta, const float* S0,
                               const int32_t* cu_seqlens, const void* out_gate, const float* norm_weight, float eps,
                               void* o, float* S_T, void* workspace, size_t workspace_bytes, void* stream) {
  if (!sp) return KDA_ERR_NULL;
  if (!A_log || !dt_bias) return KDA_ERR_NULL;
  if (!aligned(A_log, 4) || !aligned16(dt_bias)) return KDA_ERR_ALIGN;
  Epilogue ep;
  if (out_gate || norm_weight) {
    if (!out_gate || !norm_weight) return KDA_ERR_NULL;
    if (!(eps >= 0.f) || !(eps < 3.0e38f)) return KDA_ERR_ARGUMENT;
    if (!aligned16(out_gate) || !aligned16(norm_weight)) return KDA_ERR_ALIGN;
    ep.gate = out_gate;
    ep.norm_w = norm_weight;
    ep.eps = eps;
  }
  kda::StateIO io;
  io.S0 = S0;
  io.S_T = S_T;
  Producer pr;
  pr.A_log = A_log;
  pr.dt_bias = dt_bias;
  return chunk_fwd(sp, q, k, v, gate_f, beta, io, ep, pr, cu_seqlens, o, workspace, workspace_bytes, stream);
}

kda_status kda_decode_step(const kda_shape* sp, const void* q, const void* k, const void* v, const void* log_alpha,
                           const void* beta, float* S, void* o, void* stream) {
  return decode_step(sp, q, k, v, log_alpha, beta, S, nullptr, 0, o, stream);
}

kda_status kda_decode_step_slots(const kda_shape* sp, const void* q, const void* k, const void* v,
                                 const void* log_alpha, const void* beta, float* state_pool, int32_t num_slots,
                                 const int32_t* state_slots, void* o, void* stream) {
  if (!state_slots) return KDA_ERR_NULL;
  if (num_slots <= 0) return KDA_ERR_SHAPE;
  return decode_step(sp, q, k, v, log_alpha, beta, state_pool, state_slots, num_slots, o, stream);
}

kda_status kda_decode_step_layer(const kda_shape* sp, const void* q, const void* k, const void* v,
                                 const void* gate_f, const float* A_log, const float* dt_bias, const void* beta,
                                 float* state, const int32_t* state_slots, int32_t num_slots, const void* out_gate,
                                 const float* norm_weight, float eps, void* o, void* stream) {
  if (!sp) return KDA_ERR_NULL;
  if (!A_log || !dt_bias) return KDA_ERR_NULL;
  if (!aligned(A_log, 4) || !aligned(dt_bias, 4)) return KDA_ERR_ALIGN;
  if (state_slots && num_slots <= 0) return KDA_ERR_SHAPE;
  Epilogue ep;
  if (out_gate || norm_weight) {
    if (!out_gate || !norm_weight) return KDA_ERR_NULL;
    if (!(eps >= 0.f) || !(eps < 3.0e38f)) return KDA_ERR_ARGUMENT;
    if (!aligned16(out_gate) || !aligned16(norm_weight)) return KDA_ERR_ALIGN;
    ep.gate = out_gate;
    ep.norm_w = norm_weight;
    ep.eps = eps;
  }
  kda::RecProducer pr;
  pr.A_log = A_log;
  pr.dt_bias = dt_bias;
  return decode_step(sp, q, k, v, gate_f, beta, state, state_slots, state_slots ? num_slots : 0, o, stream, pr, ep);
}

kda_status kda_check_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return KDA_ERR_CUDA;
  int code = 0;
  if (cudaMemcpyFromSymbol(&code, kda::g_device_error, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
  if (code != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(kda::g_device_error, &zero, sizeof(int)) != cudaSuccess) return KDA_ERR_CUDA;
  }
  return static_cast<kda_status>(code);
}

const char* kda_status_string(kda_status status) {
  switch (status) {
    case KDA_OK: return "ok";
    case KDA_ERR_NULL: return "a required pointer is NULL";
    case KDA_ERR_SHAPE: return "invalid or inconsistent sizes";
    case KDA_ERR_DTYPE: return "unknown dtype code";
    case KDA_ERR_ALIGN: return "a pointer is not aligned as required";
    case KDA_ERR_UNSUPPORTED: return "configuration not supported (dk, dv must be 64 or 128; chunk must be 64)";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
    case KDA_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    case KDA_ERR_TIMEOUT: return "a device-side bounded wait timed out";
    case KDA_ERR_INTERNAL: return "a device-side consistency check failed";
    case KDA_ERR_ARGUMENT: return "invalid argument (cu_seqlens or flags)";
  }
  return "unknown status";
}

int32_t kda_abi_version(void) { return KDA_ABI_VERSION; }

}  // extern "C"

// ---------------------------------------------------------------------------
// kda_chunk_fwd_noalloc: kda_chunk_fwd for callers that cannot allocate device
// memory.  Its workspace is this file-scope array, reserved in the library's
// device image on every GPU that loads the library and held until the process
// exits.  Host code only ever sees a host-side stand-in for the array's name,
// so the device address is looked up with cudaGetSymbolAddress, with the
// caller's device current, on every call.  The lookup allocates nothing and
// costs a host-side table read once the module is loaded; not caching it
// means a device reset (which reloads the module at a new address) can never
// leave a stale pointer behind.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(KDA_NOALLOC_SCRATCH_BYTES);
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

kda_status noalloc_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return KDA_ERR_CUDA;
  *out = p;
  return KDA_OK;
}

}  // namespace

extern "C" kda_status kda_chunk_fwd_noalloc(const kda_shape* sp_in, const void* q, const void* k, const void* v,
                                            const void* log_alpha, const void* beta, const float* S0,
                                            const int32_t* cu_seqlens, void* o, float* S_T, void* stream) {
  const kda_status e = check_common(sp_in);
  if (e != KDA_OK) return e;
  const kda_shape* sp = sp_in;
  // an oversized request is refused before anything is launched; on the
  // pipelined path the ring is made as deep as the array allows
  const size_t need = kda_chunk_fwd_min_workspace(sp);
  if (need > kNoAllocScratchBytes) return KDA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const kda_status se = noalloc_scratch(&scratch);
    if (se != KDA_OK) return se;
  }
  return kda_chunk_fwd(sp, q, k, v, log_alpha, beta, S0, cu_seqlens, o, S_T, scratch,
                       need > 0 ? kNoAllocScratchBytes : 0, stream);
}

#ifdef KDA_TEST_HOOKS
// Test-only build: arms (1) or disarms (0) the skipped completion signal of
// g_test_skip_commit on the current device.
extern "C" int kda_test_set_skip_commit(int on) {
  return cudaMemcpyToSymbol(kda::pipe::g_test_skip_commit, &on, sizeof(int)) == cudaSuccess ? 0 : -1;
}
#endif
