// act.cuh -- per-token absmax int8 activation quantisation with an optional
// RMSNorm gain ("Key Technologies Enabling the BitNET Family": 8-bit
// activations by per-token absmax quantisation; RMSNorm without bias).
//
// Per row:  t_k = x_k * g_k (t = x without a gain),  a = max(max|t|, 1e-5),
//           q_k = clamp(rint(t_k * (127 / a)), -128, 127),
//           s = a / 127, or with a gain s = r * a / 127 where
//           r = 1 / sqrt(mean x^2 + eps) (binary64, then rounded once).
// The gain's per-row factor r cancels in the codes, so q is exact and
// independent of summation order; only s carries r.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr float kActFloor = 1e-5f;

// Block-wide reductions with a fixed combination order (deterministic and
// identical in every CTA that runs the same block size).
template <int NT>
struct RowRed {
  float f[NT / 32];
  double d[NT / 32];
  int i[NT / 32];
};

template <int NT>
__device__ __forceinline__ float block_max(float v, RowRed<NT>& r) {
  v = warp_max(v);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) r.f[w] = v;
  __syncthreads();
  float out = r.f[0];
#pragma unroll
  for (int k = 1; k < NT / 32; ++k) out = fmaxf(out, r.f[k]);
  __syncthreads();
  return out;
}

template <int NT>
__device__ __forceinline__ double block_sum_d(double v, RowRed<NT>& r) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) r.d[w] = v;
  __syncthreads();
  double out = r.d[0];
#pragma unroll
  for (int k = 1; k < NT / 32; ++k) out = __dadd_rn(out, r.d[k]);
  __syncthreads();
  return out;
}

template <int NT>
__device__ __forceinline__ int block_sum_i(int v, RowRed<NT>& r) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) r.i[w] = v;
  __syncthreads();
  int out = 0;
#pragma unroll
  for (int k = 0; k < NT / 32; ++k) out += r.i[k];
  __syncthreads();
  return out;
}

// Load 8 consecutive activations (k, k+8) of a row as binary32.
__device__ __forceinline__ void load8(const void* row, int x_dtype, int k, float (&v)[8]) {
  if (x_dtype == BITNET_BF16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(row) + k));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
      v[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(row) + k);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ void load8_gain(const float* gain, int k, float (&g)[8]) {
  const float4* p = reinterpret_cast<const float4*>(gain + k);
  const float4 a = __ldg(p), b = __ldg(p + 1);
  g[0] = a.x; g[1] = a.y; g[2] = a.z; g[3] = a.w;
  g[4] = b.x; g[5] = b.y; g[6] = b.z; g[7] = b.w;
}

__device__ __forceinline__ int quant_code(float t, float inv) {
  const float v = rintf(__fmul_rn(t, inv));
  return v >= 127.0f ? 127 : (v <= -128.0f ? -128 : static_cast<int>(v));
}

// Quantise one row (K elements, K % 16 == 0) with the whole CTA (NT
// threads).  dst receives K int8 codes (generic pointer: shared or global).
// Returns scale and code sum to every thread.
template <int NT>
__device__ void quant_row(const void* row, int x_dtype, int K, const float* __restrict__ gain, float rms_eps,
                          int8_t* dst, RowRed<NT>& red, float& scale_out, int& sum_out) {
  float amax = 0.0f;
  double ss = 0.0;
  for (int k = threadIdx.x * 8; k < K; k += NT * 8) {
    float v[8];
    load8(row, x_dtype, k, v);
    if (gain != nullptr) {
      float g[8];
      load8_gain(gain, k, g);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        amax = fmaxf(amax, fabsf(__fmul_rn(v[i], g[i])));
        ss = __dadd_rn(ss, __dmul_rn(static_cast<double>(v[i]), static_cast<double>(v[i])));
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
    }
  }
  amax = block_max<NT>(amax, red);
  if (gain != nullptr) ss = block_sum_d<NT>(ss, red);
  const float a = fmaxf(amax, kActFloor);
  const float inv = __fdiv_rn(127.0f, a);

  int qsum = 0;
  for (int k = threadIdx.x * 8; k < K; k += NT * 8) {
    float v[8];
    load8(row, x_dtype, k, v);
    if (gain != nullptr) {
      float g[8];
      load8_gain(gain, k, g);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], g[i]);
    }
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q0 = quant_code(v[i], inv), q1 = quant_code(v[i + 4], inv);
      qsum += q0 + q1;
      lo |= (static_cast<uint32_t>(q0) & 0xffu) << (8 * i);
      hi |= (static_cast<uint32_t>(q1) & 0xffu) << (8 * i);
    }
    *reinterpret_cast<uint2*>(dst + k) = make_uint2(lo, hi);
  }
  sum_out = block_sum_i<NT>(qsum, red);
  if (gain != nullptr) {
    const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(ss, static_cast<double>(K)),
                                                          static_cast<double>(rms_eps))));
    scale_out = __double2float_rn(__ddiv_rn(__dmul_rn(r, static_cast<double>(a)), 127.0));
  } else {
    scale_out = __fdiv_rn(a, 127.0f);
  }
}

constexpr int kActThreads = 256;

// One CTA per row.
__global__ void __launch_bounds__(kActThreads) quant_act_kernel(const void* __restrict__ x, int x_dtype, int K,
                                                                const float* __restrict__ gain, float rms_eps,
                                                                int8_t* __restrict__ xq, float* __restrict__ x_scale,
                                                                int32_t* __restrict__ x_sum) {
  __shared__ RowRed<kActThreads> red;
  pdl_wait();
  const int64_t m = blockIdx.x;
  const size_t esz = (x_dtype == BITNET_BF16) ? 2 : 4;
  const void* row = static_cast<const char*>(x) + m * K * esz;
  float s;
  int qs;
  quant_row<kActThreads>(row, x_dtype, K, gain, rms_eps, xq + m * K, red, s, qs);
  if (threadIdx.x == 0) {
    x_scale[m] = s;
    if (x_sum != nullptr) x_sum[m] = qs;
  }
  pdl_launch_dependents();
}

// Row sums of pre-quantised activations (when a caller gives no x_sum).
__global__ void __launch_bounds__(kActThreads) xq_rowsum_kernel(const int8_t* __restrict__ xq, int K,
                                                                int32_t* __restrict__ x_sum) {
  __shared__ RowRed<kActThreads> red;
  pdl_wait();
  const int64_t m = blockIdx.x;
  int s = 0;
  for (int k = threadIdx.x * 16; k < K; k += kActThreads * 16) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(xq + m * K + k));
    s = __dp4a(static_cast<int>(u.x), 0x01010101, s);
    s = __dp4a(static_cast<int>(u.y), 0x01010101, s);
    s = __dp4a(static_cast<int>(u.z), 0x01010101, s);
    s = __dp4a(static_cast<int>(u.w), 0x01010101, s);
  }
  s = block_sum_i<kActThreads>(s, red);
  if (threadIdx.x == 0) x_sum[m] = s;
  pdl_launch_dependents();
}

}  // namespace bitnet
