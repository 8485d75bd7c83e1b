// Output epilogue of the Kimi Linear layer as a separate pass over o: per
// (token, head) row of dv values, o <- o / sqrt(mean(o^2) + eps) * w *
// sigmoid(g).  The "Kimi Linear" summary (section on the model
// configuration) applies a per-head RMSNorm and a data-dependent output gate
// to the operator's output before the output projection.
//
// The tensor-core prefill fuses this epilogue into its output warps when its
// state CTAs have time to spare; this kernel serves the other cases (long
// sequences, where the state CTAs bound the prefill, and the CUDA-core
// paths).  It reads o and g and writes o once: HBM-bound, 3 x dv x
// sizeof(io) bytes per row.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "kda_ptx.cuh"

namespace kda {
namespace epi {

// sigmoid(g) = (1 + tanh(g / 2)) / 2 with the MUFU tanh (about 2^-11
// relative error, so the sigmoid is within ~2.5e-4 absolute)
__device__ __forceinline__ float sigmoid_tanh(float g) { return fmaf(0.5f, tanh_approx(0.5f * g), 0.5f); }

template <typename TO>
struct Vec8;  // 8 consecutive values of a row
template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[8]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    __stcs(reinterpret_cast<uint4*>(p), make_uint4(w[0], w[1], w[2], w[3]));
  }
};
template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&x)[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x, x[1] = a.y, x[2] = a.z, x[3] = a.w, x[4] = b.x, x[5] = b.y, x[6] = b.z, x[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&x)[8]) {
    __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
    __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(x[4], x[5], x[6], x[7]));
  }
};

constexpr int kThreads = 256;

// One row of DV values per DV/8 lanes (8 values a lane); a warp covers
// 256/DV rows per step and each thread handles two rows per iteration.  The
// loop bound is warp-uniform so that every lane joins the shuffles.
template <typename TO, int DV>
__global__ void __launch_bounds__(kThreads) kda_output_gate_kernel(TO* __restrict__ o, const TO* __restrict__ g,
                                                                   const float* __restrict__ w, float eps,
                                                                   int64_t rows) {
  constexpr int LPR = DV / 8;         // lanes per row
  constexpr int RPW = 32 / LPR;       // rows per warp step
  const int lane = threadIdx.x & 31;
  const int sub = lane / LPR, c0 = (lane % LPR) * 8;
  float wr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) wr[i] = __ldg(w + c0 + i);
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const int64_t stride = warps * RPW;
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5)) * RPW; base < rows;
       base += 2 * stride) {
    const int64_t r0 = base + sub, r1 = base + stride + sub;
    const bool v0 = r0 < rows, v1 = r1 < rows;
    float x0[8] = {}, x1[8] = {}, g0[8] = {}, g1[8] = {};
    if (v0) {
      Vec8<TO>::load(o + r0 * DV + c0, x0);
      Vec8<TO>::load(g + r0 * DV + c0, g0);
    }
    if (v1) {
      Vec8<TO>::load(o + r1 * DV + c0, x1);
      Vec8<TO>::load(g + r1 * DV + c0, g1);
    }
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      s0 = fmaf(x0[i], x0[i], s0);
      s1 = fmaf(x1[i], x1[i], s1);
    }
#pragma unroll
    for (int m = LPR / 2; m >= 1; m >>= 1) {
      s0 += __shfl_xor_sync(0xffffffffu, s0, m);
      s1 += __shfl_xor_sync(0xffffffffu, s1, m);
    }
    const float rinv0 = rsqrtf(s0 * (1.f / DV) + eps), rinv1 = rsqrtf(s1 * (1.f / DV) + eps);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x0[i] = x0[i] * rinv0 * wr[i] * sigmoid_tanh(g0[i]);
      x1[i] = x1[i] * rinv1 * wr[i] * sigmoid_tanh(g1[i]);
    }
    if (v0) Vec8<TO>::store(o + r0 * DV + c0, x0);
    if (v1) Vec8<TO>::store(o + r1 * DV + c0, x1);
  }
}

}  // namespace epi
}  // namespace kda
