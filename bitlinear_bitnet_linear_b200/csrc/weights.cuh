// weights.cuh -- offline weight preparation: exact absmean scale, ternary
// rounding, 2-bit pack and unpack.
//
// Absmean ternarisation follows "Key Technologies Enabling the BitNET
// Family" (Advanced Quantization Methodologies: absmean ternary weights)
// and "BitNet / Ternary / Binary -- Les LLMs 1-bit" (BitLinear forward:
// beta = mean|w|, clamp(round(w / (beta + 1e-8)), -1, 1)).  The 2-bit
// layout is this library's (2 bits per weight: "BitNet Technical Notes").
#pragma once

#include "common.cuh"

namespace bitnet {

// ---------------------------------------------------------------------------
// Exact sum of |W|.
//
// Every finite binary32 magnitude is an integer multiple of 2^-149:
//   |w| = M * 2^(E - 150),  M = 2^23 + mantissa (E >= 1) or mantissa with
//   E := 1 (subnormal).
// Split E = 16b + r.  Bin b accumulates M << r (< 2^39) in a uint64; a block
// handles at most 2^24 elements, so a bin cannot overflow.  The per-block
// bins are integers, so the final total does not depend on the order of
// accumulation: gamma is deterministic for any launch shape.
// ---------------------------------------------------------------------------
constexpr int kAbsThreads = 256;
constexpr int kAbsBins = 16;
constexpr int64_t kAbsMaxPerBlock = int64_t(1) << 24;

__device__ __forceinline__ void abs_bin_add(uint64_t* my_bins /* stride kAbsThreads */, float v, bool& bad) {
  uint32_t bits = __float_as_uint(v) & 0x7fffffffu;
  uint32_t e = bits >> 23;
  uint32_t m = bits & 0x7fffffu;
  if (e == 255u) { bad = true; return; }
  if (e == 0u) {
    if (m == 0u) return;
    e = 1u;
  } else {
    m |= 0x800000u;
  }
  my_bins[(e >> 4) * kAbsThreads] += static_cast<uint64_t>(m) << (e & 15u);
}

__global__ void __launch_bounds__(kAbsThreads) absmean_partial_kernel(const float* __restrict__ W, int64_t n,
                                                                      int64_t per_block,
                                                                      uint64_t* __restrict__ partial,
                                                                      uint32_t* status) {
  __shared__ uint64_t bins[kAbsBins * kAbsThreads];
  const int tid = threadIdx.x;
  for (int b = 0; b < kAbsBins; ++b) bins[b * kAbsThreads + tid] = 0;
  uint64_t* mine = bins + tid;
  bool bad = false;

  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * per_block;
  const int64_t b1 = min(n, b0 + per_block);
  // per_block and n are multiples of 16, W is 16-byte aligned: float4 loads.
  const float4* W4 = reinterpret_cast<const float4*>(W);
  for (int64_t i = b0 / 4 + tid; i < b1 / 4; i += kAbsThreads) {
    float4 v = __ldg(W4 + i);
    abs_bin_add(mine, v.x, bad);
    abs_bin_add(mine, v.y, bad);
    abs_bin_add(mine, v.z, bad);
    abs_bin_add(mine, v.w, bad);
  }
  if (bad) record_error(status, BITNET_ERR_VALUE, 0x101u);
  __syncthreads();
  const int warp = tid >> 5, lane = tid & 31;
  for (int b = warp; b < kAbsBins; b += kAbsThreads / 32) {
    uint64_t s = 0;
    for (int t = lane; t < kAbsThreads; t += 32) s += bins[b * kAbsThreads + t];
    s = warp_sum<unsigned long long>(s);
    if (lane == 0) partial[static_cast<int64_t>(blockIdx.x) * kAbsBins + b] = s;
  }
}

// 256 threads: sum the per-block bins (16 threads per bin, exact in 128
// bits), then one thread assembles the exact total in a 384-bit integer
// (units of 2^-150), rounds it once to binary64, divides by n in binary64 and
// rounds to binary32.
constexpr int kAbsFinThreads = 256;
__global__ void __launch_bounds__(kAbsFinThreads) absmean_finalize_kernel(const uint64_t* __restrict__ partial,
                                                                          int nblocks, int64_t n,
                                                                          float* __restrict__ gamma_out) {
  __shared__ unsigned long long plo[16][kAbsBins], phi[16][kAbsBins];
  __shared__ unsigned long long lo_s[kAbsBins], hi_s[kAbsBins];
  const int tid = threadIdx.x;
  {
    const int bin = tid & (kAbsBins - 1), part = tid >> 4;
    unsigned __int128 s = 0;
    for (int b = part; b < nblocks; b += kAbsFinThreads / kAbsBins)
      s += partial[static_cast<int64_t>(b) * kAbsBins + bin];
    plo[part][bin] = static_cast<unsigned long long>(s);
    phi[part][bin] = static_cast<unsigned long long>(s >> 64);
  }
  __syncthreads();
  if (tid < kAbsBins) {
    unsigned __int128 s = 0;
    for (int part = 0; part < kAbsFinThreads / kAbsBins; ++part)
      s += (static_cast<unsigned __int128>(phi[part][tid]) << 64) | plo[part][tid];
    lo_s[tid] = static_cast<unsigned long long>(s);
    hi_s[tid] = static_cast<unsigned long long>(s >> 64);
  }
  __syncthreads();
  if (tid != 0) return;

  uint64_t limb[6] = {0, 0, 0, 0, 0, 0};
  for (int b = 0; b < kAbsBins; ++b) {
    // add (hi:lo) << 16b
    const int sh = 16 * b, li = sh >> 6, off = sh & 63;
    const uint64_t lo = lo_s[b], hi = hi_s[b];
    uint64_t w[3];
    w[0] = lo << off;
    w[1] = (off ? (lo >> (64 - off)) : 0ull) | (hi << off);
    w[2] = off ? (hi >> (64 - off)) : 0ull;
    uint64_t carry = 0;
    for (int t = 0; li + t < 6; ++t) {
      const uint64_t add = (t < 3 ? w[t] : 0ull);
      const uint64_t s1 = limb[li + t] + add;
      const uint64_t c1 = s1 < add ? 1ull : 0ull;
      const uint64_t s2 = s1 + carry;
      const uint64_t c2 = s2 < carry ? 1ull : 0ull;
      limb[li + t] = s2;
      carry = c1 + c2;
      if (t >= 2 && carry == 0) break;
    }
  }
  int top = -1;
  for (int i = 5; i >= 0; --i)
    if (limb[i]) { top = i; break; }
  double total;
  if (top < 0) {
    total = 0.0;
  } else {
    const int p = 64 * top + (63 - __clzll(static_cast<long long>(limb[top])));
    if (p < 64) {
      total = scalbn(__ull2double_rn(limb[0]), -150);
    } else {
      const int lob = p - 63;          // keep bits [lob, lob + 63]
      const int li = lob >> 6, off = lob & 63;
      uint64_t word = limb[li] >> off;
      if (off && li + 1 < 6) word |= limb[li + 1] << (64 - off);
      bool sticky = (off != 0) && ((limb[li] & ((1ull << off) - 1ull)) != 0);
      for (int i = 0; i < li; ++i) sticky = sticky || (limb[i] != 0);
      if (sticky) word |= 1ull;
      total = scalbn(__ull2double_rn(word), lob - 150);
    }
  }
  const double mean = __ddiv_rn(total, static_cast<double>(n));
  *gamma_out = __double2float_rn(mean);
}

// ---------------------------------------------------------------------------
// Ternary rounding: q = clamp(rint(w / (gamma + eps)), -1, 1), binary32.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int8_t ternary_of(float w, float d) {
  const float r = rintf(__fdiv_rn(w, d));
  return r >= 1.0f ? int8_t(1) : (r <= -1.0f ? int8_t(-1) : int8_t(0));
}

__global__ void __launch_bounds__(256) ternarise_kernel(const float* __restrict__ W, int64_t n4,
                                                        const float* __restrict__ gamma, float eps,
                                                        int8_t* __restrict__ Wq) {
  const float d = __fadd_rn(*gamma, eps);
  const float4* W4 = reinterpret_cast<const float4*>(W);
  char4* Q4 = reinterpret_cast<char4*>(Wq);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(W4 + i);
    char4 q;
    q.x = ternary_of(v.x, d);
    q.y = ternary_of(v.y, d);
    q.z = ternary_of(v.z, d);
    q.w = ternary_of(v.w, d);
    Q4[i] = q;
  }
}

// ---------------------------------------------------------------------------
// 2-bit pack / unpack.  One thread per 16-weight group (one 32-bit word):
// weight k = 16g + 4s + j at bits [8j + 2s, 8j + 2s + 1], code = q + 1.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pack_kernel(const int8_t* __restrict__ Wq, int64_t ngroups,
                                                   uint32_t* __restrict__ Wp, uint32_t* n_invalid) {
  uint32_t bad = 0;
  const uint4* Q = reinterpret_cast<const uint4*>(Wq);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < ngroups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(Q + g);
    const uint32_t in[4] = {v.x, v.y, v.z, v.w};   // in[s] byte j = q[16g + 4s + j]
    uint32_t word = 0;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q = static_cast<int8_t>((in[s] >> (8 * j)) & 0xffu);
        uint32_t c;
        if (q >= -1 && q <= 1) {
          c = static_cast<uint32_t>(q + 1);
        } else {
          c = 3u;
          ++bad;
        }
        word |= c << (8 * j + 2 * s);
      }
    }
    Wp[g] = word;
  }
  if (n_invalid != nullptr && bad) atomicAdd(n_invalid, bad);
}

__global__ void __launch_bounds__(256) unpack_kernel(const uint32_t* __restrict__ Wp, int64_t ngroups,
                                                     int8_t* __restrict__ Wq, uint32_t* n_invalid) {
  uint32_t bad = 0;
  uint4* Q = reinterpret_cast<uint4*>(Wq);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < ngroups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t word = __ldg(Wp + g);
    uint32_t out[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      uint32_t o = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t c = (word >> (8 * j + 2 * s)) & 3u;
        int q;
        if (c == 3u) {
          q = 0;
          ++bad;
        } else {
          q = static_cast<int>(c) - 1;
        }
        o |= (static_cast<uint32_t>(q) & 0xffu) << (8 * j);
      }
      out[s] = o;
    }
    Q[g] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (n_invalid != nullptr && bad) atomicAdd(n_invalid, bad);
}

// Empty kernel launched WITHOUT programmatic serialisation after calls that
// write weights: a following GEMV may read weights before its dependency
// wait, so the weight writer must be fully complete first.
// BitNet b1 ("BitNet / Ternary / Binary", BitNet b1 (binaire): every weight
// exactly +1 or -1): W_b = +1 where W >= 0, else -1 (NaN gives -1).
__global__ void __launch_bounds__(256) binarise_kernel(const float* __restrict__ W, int64_t n4,
                                                       int8_t* __restrict__ Wb) {
  const float4* W4 = reinterpret_cast<const float4*>(W);
  char4* B4 = reinterpret_cast<char4*>(Wb);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(W4 + i);
    char4 b;
    b.x = v.x >= 0.0f ? 1 : -1;
    b.y = v.y >= 0.0f ? 1 : -1;
    b.z = v.z >= 0.0f ? 1 : -1;
    b.w = v.w >= 0.0f ? 1 : -1;
    B4[i] = b;
  }
}

// 1-bit pack: one uint32 per 32 weights, weight 32g + 4s + j at bit 8j + s
// (bit 1 for +1).  Values other than +-1 are stored as 0 and counted.
__global__ void __launch_bounds__(256) pack_b1_kernel(const int8_t* __restrict__ Wb, int64_t ngroups,
                                                      uint32_t* __restrict__ Wp, uint32_t* n_invalid) {
  uint32_t bad = 0;
  const uint4* Q = reinterpret_cast<const uint4*>(Wb);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < ngroups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 a = __ldg(Q + 2 * g), b = __ldg(Q + 2 * g + 1);
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};   // in[s] byte j = w[32g + 4s + j]
    uint32_t word = 0;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int v = static_cast<int8_t>((in[s] >> (8 * j)) & 0xffu);
        if (v == 1)
          word |= 1u << (8 * j + s);
        else if (v != -1)
          ++bad;
      }
    }
    Wp[g] = word;
  }
  if (n_invalid != nullptr && bad) atomicAdd(n_invalid, bad);
}

__global__ void __launch_bounds__(256) unpack_b1_kernel(const uint32_t* __restrict__ Wp, int64_t ngroups,
                                                        int8_t* __restrict__ Wb) {
  uint4* Q = reinterpret_cast<uint4*>(Wb);
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < ngroups;
       g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t word = __ldg(Wp + g);
    uint32_t out[8];
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      // bits (word >> s) & 0x01010101 are the weights 32g + 4s .. + 3: 1 -> +1, 0 -> -1 (0xff)
      const uint32_t bits = (word >> s) & 0x01010101u;
      out[s] = bits | ((0x01010101u - bits) * 0xffu);
    }
    Q[2 * g] = make_uint4(out[0], out[1], out[2], out[3]);
    Q[2 * g + 1] = make_uint4(out[4], out[5], out[6], out[7]);
  }
}

// Base-3 pack: five ternary weights per byte (3^5 = 243 <= 256).  Row n
// takes row_bytes = ceil(K/80)*16 bytes; byte j of the uint32 group g holds
// sum_i c(20g + 4i + j) 3^i, i = 0..4, with codes c = q + 1 (weights past K:
// code 1).  Values outside {-1, 0, 1} are stored as code 1 and counted.
// One thread per group.
__global__ void __launch_bounds__(256) pack_t3_kernel(const int8_t* __restrict__ Wq, int64_t N, int64_t K,
                                                      int64_t row_bytes, uint32_t* __restrict__ Wp,
                                                      uint32_t* n_invalid) {
  uint32_t bad = 0;
  const int64_t gpr = row_bytes / 4, total = N * gpr;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = t / gpr, g = t - n * gpr;
    const int8_t* row = Wq + n * K;
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t v = 0, p3 = 1;
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const int64_t k = 20 * g + 4 * i + j;
        uint32_t c = 1;
        if (k < K) {
          const int q = row[k];
          if (q >= -1 && q <= 1)
            c = static_cast<uint32_t>(q + 1);
          else
            ++bad;
        }
        v += c * p3;
        p3 *= 3u;
      }
      word |= v << (8 * j);
    }
    Wp[t] = word;
  }
  if (n_invalid != nullptr && bad) atomicAdd(n_invalid, bad);
}

// Inverse of pack_t3_kernel for k < K; a byte above 242 is invalid: its
// weights read as 0 and it is counted.
__global__ void __launch_bounds__(256) unpack_t3_kernel(const uint32_t* __restrict__ Wp, int64_t N, int64_t K,
                                                        int64_t row_bytes, int8_t* __restrict__ Wq,
                                                        uint32_t* n_invalid) {
  uint32_t bad = 0;
  const int64_t gpr = row_bytes / 4, total = N * gpr;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = t / gpr, g = t - n * gpr;
    const uint32_t word = __ldg(Wp + t);
    int8_t* row = Wq + n * K;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t v = (word >> (8 * j)) & 0xffu;
      const bool valid = v <= 242u;
      if (!valid && 20 * g + j < K) ++bad;
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const int64_t k = 20 * g + 4 * i + j;
        const uint32_t c = v % 3u;
        v /= 3u;
        if (k < K) row[k] = valid ? static_cast<int8_t>(static_cast<int>(c) - 1) : static_cast<int8_t>(0);
      }
    }
  }
  if (n_invalid != nullptr && bad) atomicAdd(n_invalid, bad);
}

__global__ void stream_fence_kernel() {}

}  // namespace bitnet
