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

// Scratch for quant_rows: per-warp partials of up to MT rows.
template <int NT, int MT>
struct QuantScratch {
  float amax[MT][NT / 32];
  double ss[MT][NT / 32];
  int qpart[MT][NT / 32];
};

__device__ __forceinline__ void decode8(const uint4 (&raw)[2], int x_dtype, float (&v)[8]) {
  if (x_dtype == BITNET_BF16) {
    const uint32_t w[4] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_bits_to_float(w[i] & 0xffffu);
      v[2 * i + 1] = bf16_bits_to_float(w[i] >> 16);
    }
  } else {
    v[0] = __uint_as_float(raw[0].x); v[1] = __uint_as_float(raw[0].y);
    v[2] = __uint_as_float(raw[0].z); v[3] = __uint_as_float(raw[0].w);
    v[4] = __uint_as_float(raw[1].x); v[5] = __uint_as_float(raw[1].y);
    v[6] = __uint_as_float(raw[1].z); v[7] = __uint_as_float(raw[1].w);
  }
}

template <bool SMEM_SRC = false>
__device__ __forceinline__ void load8raw(const char* row, int x_dtype, int k, uint4 (&raw)[2]) {
  if (x_dtype == BITNET_BF16) {
    const uint4* q = reinterpret_cast<const uint4*>(row + 2 * static_cast<int64_t>(k));
    raw[0] = SMEM_SRC ? *q : __ldg(q);
  } else {
    const uint4* q = reinterpret_cast<const uint4*>(row + 4 * static_cast<int64_t>(k));
    raw[0] = SMEM_SRC ? q[0] : __ldg(q);
    raw[1] = SMEM_SRC ? q[1] : __ldg(q + 1);
  }
}

// Block (or named-barrier group) synchronisation used by quant_rows.
// BAR == 0: __syncthreads; otherwise named barrier BAR over NT threads.
template <int BAR, int NT>
__device__ __forceinline__ void group_sync() {
  if constexpr (BAR == 0)
    __syncthreads();
  else
    asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

// Byte offset of activation k inside a 64-byte chunk row with the 16-byte
// slots XOR-swizzled by chunk index: lanes that read consecutive chunks hit
// distinct bank groups.
__device__ __forceinline__ int xs_swizzle(int k) {
  const int c = k >> 6, g = (k >> 4) & 3;
  return (c << 6) | ((g ^ ((c >> 1) & 3)) << 4) | (k & 15);
}

// Byte offset of activation k in the block-permuted code row used by the
// 16-byte streaming GEMV (K % 64 == 0): the 16-byte block g = 4c + e (codes
// 16g .. 16g + 15) is stored at e * K/4 + 16 c, so the four blocks that meet
// one 16-byte load of packed weights (64 weights, chunk c) sit K/4 bytes
// apart and consecutive chunks are consecutive in each quarter.
__device__ __forceinline__ int xs_blocked(int k, int K) {
  const int g = k >> 4;
  return (g & 3) * (K >> 2) + ((g >> 2) << 4) + (k & 15);
}

// The same with eight quarters, for the 1-bit GEMV (K % 128 == 0): 16-byte
// block g = 8c + e at e * K/8 + 16 c, the eight blocks that meet one 16-byte
// load of packed signs (128 weights, chunk c).
__device__ __forceinline__ int xs_blocked8(int k, int K) {
  const int g = k >> 4;
  return (g & 7) * (K >> 3) + ((g >> 3) << 4) + (k & 15);
}

// ReLU^2 gate of the feed-forward layers: the down projection's input is
// t = max(g, 0)^2 * u for the gate and up projections' outputs g and u, in
// binary32 with one rounding per operation: (r * r) * u.  v holds g on entry.
template <bool SMEM_SRC = false>
__device__ __forceinline__ void relu2_gate8(const char* up_row, int x_dtype, int k, float (&v)[8]) {
  uint4 raw[2];
  load8raw<SMEM_SRC>(up_row, x_dtype, k, raw);
  float u[8];
  decode8(raw, x_dtype, u);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float r = fmaxf(v[i], 0.0f);
    v[i] = __fmul_rn(__fmul_rn(r, r), u[i]);
  }
}

// Quantise rows 0..M-1 (M <= MT, K % 16 == 0) with one CTA of NT
// threads.  Pass 1 finds max|t| (and sum x^2 with a gain) per row, keeping
// up to C 8-element bfloat16 chunks per thread in registers; one
// __syncthreads combines the per-warp partials in a fixed order.  Pass 2
// writes the codes to dst (row stride dst_stride, generic address) and
// leaves per-warp partial code sums in S.qpart: the caller's next
// __syncthreads publishes both.  scale[m] is returned to every thread.
// The group is threads [tid_base, tid_base + NT) of the block.  With x2
// (same layout as x), the input is the ReLU^2 gate of x (gate) and x2 (up).
template <int NT, int MT, int C, bool SMEM_SRC = false, int BAR = 0, bool SWZ = false>
__device__ __forceinline__ void quant_rows(const char* __restrict__ x, int x_dtype, int64_t row_bytes, int M,
                                           int K, const float* __restrict__ gain, float rms_eps, int8_t* dst,
                                           int64_t dst_stride, QuantScratch<NT, MT>& S, float (&scale)[MT],
                                           int tid_base = 0, int blocked = 0,
                                           const char* __restrict__ x2 = nullptr) {
  const int tid = static_cast<int>(threadIdx.x) - tid_base, lane = tid & 31, warp = tid >> 5;
  const bool cache_ok = (x_dtype == BITNET_BF16) && x2 == nullptr;
  uint4 cache[MT][C];
  float am[MT];
  double ss[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    am[m] = 0.0f;
    ss[m] = 0.0;
    if (m < M) {
      const char* row = x + m * row_bytes;
      auto process = [&](const float (&v)[8], int k) {
        if (gain != nullptr) {
          float g[8];
          load8_gain(gain, k, g);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            am[m] = fmaxf(am[m], fabsf(__fmul_rn(v[i], g[i])));
            ss[m] = __dadd_rn(ss[m], __dmul_rn(static_cast<double>(v[i]), static_cast<double>(v[i])));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) am[m] = fmaxf(am[m], fabsf(v[i]));
        }
      };
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const int k = (c * NT + tid) * 8;
        if (k < K) {
          uint4 raw[2];
          load8raw<SMEM_SRC>(row, x_dtype, k, raw);
          if (cache_ok) cache[m][c] = raw[0];
          float v[8];
          decode8(raw, x_dtype, v);
          if (x2 != nullptr) relu2_gate8<SMEM_SRC>(x2 + m * row_bytes, x_dtype, k, v);
          process(v, k);
        }
      }
#pragma unroll 4
      for (int k = (C * NT + tid) * 8; k < K; k += NT * 8) {
        uint4 raw[2];
        load8raw<SMEM_SRC>(row, x_dtype, k, raw);
        float v[8];
        decode8(raw, x_dtype, v);
        if (x2 != nullptr) relu2_gate8<SMEM_SRC>(x2 + m * row_bytes, x_dtype, k, v);
        process(v, k);
      }
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    am[m] = warp_max(am[m]);
    if (gain != nullptr) ss[m] = warp_sum(ss[m]);
    if (lane == 0) {
      S.amax[m][warp] = am[m];
      S.ss[m][warp] = ss[m];
    }
  }
  group_sync<BAR, NT>();
  float inv[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    float A = S.amax[m][0];
    double SS = S.ss[m][0];
#pragma unroll
    for (int w = 1; w < NT / 32; ++w) {
      A = fmaxf(A, S.amax[m][w]);
      SS = __dadd_rn(SS, S.ss[m][w]);
    }
    const float a = fmaxf(A, kActFloor);
    inv[m] = __fdiv_rn(127.0f, a);
    if (gain != nullptr) {
      const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(__ddiv_rn(SS, static_cast<double>(K)),
                                                            static_cast<double>(rms_eps))));
      scale[m] = __double2float_rn(__ddiv_rn(__dmul_rn(r, static_cast<double>(a)), 127.0));
    } else {
      scale[m] = __fdiv_rn(a, 127.0f);
    }
  }
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    int qs = 0;
    if (m < M) {
      const char* row = x + m * row_bytes;
      int8_t* drow = dst + m * dst_stride;
      auto emit = [&](float (&v)[8], int k) {
        if (gain != nullptr) {
          float g[8];
          load8_gain(gain, k, g);
#pragma unroll
          for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], g[i]);
        }
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int q0 = quant_code(v[i], inv[m]), q1 = quant_code(v[i + 4], inv[m]);
          qs += q0 + q1;
          lo |= (static_cast<uint32_t>(q0) & 0xffu) << (8 * i);
          hi |= (static_cast<uint32_t>(q1) & 0xffu) << (8 * i);
        }
        const int off = SWZ ? xs_swizzle(k) : (blocked == 1 ? xs_blocked(k, K) : (blocked == 2 ? xs_blocked8(k, K) : k));
        *reinterpret_cast<uint2*>(drow + off) = make_uint2(lo, hi);
      };
#pragma unroll
      for (int c = 0; c < C; ++c) {
        const int k = (c * NT + tid) * 8;
        if (k < K) {
          uint4 raw[2];
          if (cache_ok)
            raw[0] = cache[m][c];
          else
            load8raw<SMEM_SRC>(row, x_dtype, k, raw);
          float v[8];
          decode8(raw, x_dtype, v);
          if (x2 != nullptr) relu2_gate8<SMEM_SRC>(x2 + m * row_bytes, x_dtype, k, v);
          emit(v, k);
        }
      }
#pragma unroll 4
      for (int k = (C * NT + tid) * 8; k < K; k += NT * 8) {
        uint4 raw[2];
        load8raw<SMEM_SRC>(row, x_dtype, k, raw);
        float v[8];
        decode8(raw, x_dtype, v);
        if (x2 != nullptr) relu2_gate8<SMEM_SRC>(x2 + m * row_bytes, x_dtype, k, v);
        emit(v, k);
      }
    }
    qs = warp_sum(qs);
    if (lane == 0) S.qpart[m][warp] = qs;
  }
}

constexpr int kActThreads = 256;

// One CTA per row.
// With x2: quantise the ReLU^2 gate of x (gate) and x2 (up).
__global__ void __launch_bounds__(kActThreads) quant_act_kernel(const void* __restrict__ x, int x_dtype, int K,
                                                                const float* __restrict__ gain, float rms_eps,
                                                                int8_t* __restrict__ xq, float* __restrict__ x_scale,
                                                                int32_t* __restrict__ x_sum,
                                                                const void* __restrict__ x2) {
  __shared__ QuantScratch<kActThreads, 1> S;
  pdl_launch_dependents();
  pdl_wait();
  const int64_t m = blockIdx.x;
  const int64_t esz = (x_dtype == BITNET_BF16) ? 2 : 4;
  float sc[1];
  quant_rows<kActThreads, 1, 2>(static_cast<const char*>(x) + m * K * esz, x_dtype, K * esz, 1, K, gain, rms_eps,
                                xq + m * K, K, S, sc, 0, 0,
                                x2 != nullptr ? static_cast<const char*>(x2) + m * K * esz : nullptr);
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
#pragma unroll
    for (int w = 0; w < kActThreads / 32; ++w) t += S.qpart[0][w];
    x_scale[m] = sc[0];
    if (x_sum != nullptr) x_sum[m] = t;
  }
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
