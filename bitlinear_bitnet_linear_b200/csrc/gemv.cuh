// gemv.cuh -- packed-ternary GEMV for a few tokens (decode).
//
// y[m,n] = (sum_k x_q[m,k] * W_q[n,k]) * gamma * s_x[m]      (M <= 4)
//
// The ternary dot product ("sum of activations where the weight is +1 minus
// the sum where it is -1", Hacker News thread on the b1.58 paper) is formed
// from the stored codes c = q + 1 in {0, 1, 2}:
//     sum_k q_k x_k = sum_k c_k x_k - sum_k x_k,
// so the 2-bit fields feed dp4a (unsigned codes x signed int8) directly:
// masking field s of a packed 32-bit group (mask 0x03030303 << 2s) leaves
// four codes scaled by 4^s lined up with four consecutive activations, and
// four per-field accumulators are rescaled by exact shifts at the end.
//
// Design for B200:
//   * each CTA owns a contiguous slab of rows, which is one contiguous byte
//     range of the packed matrix; it is streamed into shared memory with
//     cp.async.bulk (TMA, no multicast) in stages tracked by mbarriers;
//   * the first stages are issued BEFORE griddepcontrol.wait, so under
//     programmatic dependent launch the weight stream of this call overlaps
//     the tail of the previous kernel (weights never depend on it);
//   * the activation row(s) are quantised by every CTA in its prologue
//     (fused quantiser) straight into shared memory, then reused from there
//     for all rows of the slab.
#pragma once

#include "act.cuh"
#include "common.cuh"

namespace bitnet {

constexpr int kGvThreads = 256;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGvMaxStages = 8;
constexpr int kGvHeader = 1024;   // barriers + reduction scratch + per-token scale

struct GemvParams {
  // activations: either raw x (fused quantiser) or pre-quantised x_q
  const void* x;
  int x_dtype;
  const float* gain;
  float rms_eps;
  const int8_t* xq;
  const float* x_scale;
  // weights
  const uint8_t* Wp;
  const float* gamma;
  // outputs
  void* y;
  int y_dtype;
  int32_t* acc;
  // shapes and partition
  int M, K, N;
  int rows_base, rows_extra;   // CTA b owns rows_base + (b < rows_extra) rows
  int Kp;                      // K rounded up to 64: x_q row stride in shared memory
  int wrow;                    // shared bytes per weight row (K/4 rounded up to 16)
  int stage_rows, stages;      // ring of `stages` buffers of `stage_rows` rows
  int bulk;                    // 1: weights via cp.async.bulk (K % 64 == 0)
  uint64_t limit_ns;
  uint32_t* status;
};

template <int MT>
struct GemvHeader {
  uint64_t full[kGvMaxStages];
  QuantScratch<kGvThreads, MT> q;
  float scale[MT];
};

template <int MT, int R, bool FUSED>
__global__ void __launch_bounds__(kGvThreads) gemv_kernel(const GemvParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  static_assert(sizeof(GemvHeader<MT>) <= kGvHeader, "header too large");
  GemvHeader<MT>& H = *reinterpret_cast<GemvHeader<MT>*>(smem);
  int8_t* xs = reinterpret_cast<int8_t*>(smem + kGvHeader);
  uint8_t* ring = smem + kGvHeader + MT * p.Kp;   // MT * Kp is a multiple of 64; header 1024

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x;
  const int cnt = p.rows_base + (b < p.rows_extra ? 1 : 0);
  const int64_t n0 = static_cast<int64_t>(b) * p.rows_base + min(b, p.rows_extra);
  const int nst = (cnt + p.stage_rows - 1) / p.stage_rows;
  const int64_t rowbytes = p.K / 4;
  const int stage_bytes = p.stage_rows * p.wrow;

  auto issue = [&](int i) {   // one thread: bulk-copy stage i into ring slot i % stages
    const int s = i % p.stages;
    const int r0 = i * p.stage_rows;
    const int rc = min(p.stage_rows, cnt - r0);
    const uint32_t bytes = static_cast<uint32_t>(rc * rowbytes);
    mbar_expect_tx(&H.full[s], bytes);
    bulk_g2s(ring + s * stage_bytes, p.Wp + (n0 + r0) * rowbytes, bytes, &H.full[s]);
  };

  // Weights never depend on earlier kernels: start streaming them at once.
  // The first __syncthreads below orders this initialisation before any
  // other thread waits on the barriers.
  if (tid == 0 && p.bulk) {
    for (int s = 0; s < p.stages; ++s) mbar_init(&H.full[s], 1);
    fence_mbar_init();
    for (int i = 0; i < min(p.stages, nst); ++i) issue(i);
  }
  // Let the next kernel in the stream launch and start its own weight
  // stream; it still waits for this grid before touching our outputs.
  pdl_launch_dependents();
  pdl_wait();

  // ---- prologue: activation codes into shared memory, zero padded --------
  if constexpr (FUSED) {
    const int64_t esz = (p.x_dtype == BITNET_BF16) ? 2 : 4;
    float sc[MT];
    quant_rows<kGvThreads, MT, (MT == 1 ? 4 : (MT == 2 ? 2 : 1))>(static_cast<const char*>(p.x), p.x_dtype,
                                                                 p.K * esz, p.M, p.K, p.gain, p.rms_eps, xs, p.Kp,
                                                                 H.q, sc);
    if (tid == 0) {
#pragma unroll
      for (int m = 0; m < MT; ++m) H.scale[m] = sc[m];
    }
  } else {
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int part = 0;
      if (m < p.M) {
        for (int k = tid * 16; k < p.K; k += kGvThreads * 16) {
          const uint4 u = __ldg(reinterpret_cast<const uint4*>(p.xq + static_cast<int64_t>(m) * p.K + k));
          *reinterpret_cast<uint4*>(xs + m * p.Kp + k) = u;
          part = __dp4a(static_cast<int>(u.x), 0x01010101, part);
          part = __dp4a(static_cast<int>(u.y), 0x01010101, part);
          part = __dp4a(static_cast<int>(u.z), 0x01010101, part);
          part = __dp4a(static_cast<int>(u.w), 0x01010101, part);
        }
      }
      part = warp_sum(part);
      if (lane == 0) H.q.qpart[m][warp] = part;
      if (tid == 0) H.scale[m] = (m < p.M) ? __ldg(p.x_scale + m) : 0.0f;
    }
  }
  for (int m = 0; m < MT; ++m) {
    const int k0 = (m < p.M) ? p.K : 0;
    for (int k = k0 + tid * 16; k < p.Kp; k += kGvThreads * 16)
      *reinterpret_cast<uint4*>(xs + m * p.Kp + k) = make_uint4(0, 0, 0, 0);
    if (m >= p.M && lane == 0) H.q.qpart[m][warp] = 0;
  }
  __syncthreads();

  const float gamma = __ldg(p.gamma);
  const int nchunk = p.Kp / 64;   // 16-byte chunks (64 weights) per row
  bool failed = false;

  for (int i = 0; i < nst; ++i) {
    const int s = i % p.stages;
    const int r0 = i * p.stage_rows;
    const int rc = min(p.stage_rows, cnt - r0);
    uint8_t* buf = ring + s * stage_bytes;
    if (p.bulk) {
      const bool ok = mbar_wait_bounded(&H.full[s], static_cast<uint32_t>((i / p.stages) & 1), p.limit_ns, nullptr);
      // CTA-uniform decision: every thread leaves together or none does.
      failed = __syncthreads_or(ok ? 0 : 1) != 0;
      if (failed && tid == 0) record_error(p.status, BITNET_ERR_TIMEOUT, 0x201u);
    } else {
      // K % 64 != 0: rows are 4-byte aligned only; copy with word loads
      // into 16-byte-aligned padded rows.
      const int wpr = p.K / 16;   // 32-bit words per row
      for (int t = tid; t < rc * wpr; t += kGvThreads) {
        const int r = t / wpr, w = t - r * wpr;
        const uint32_t v =
            __ldg(reinterpret_cast<const uint32_t*>(p.Wp + (n0 + r0 + r) * rowbytes) + w);
        reinterpret_cast<uint32_t*>(buf + r * p.wrow)[w] = v;
      }
      __syncthreads();
    }
    if (failed) break;

    const int wstride = p.bulk ? static_cast<int>(rowbytes) : p.wrow;
    for (int rg = warp; rg * R < rc; rg += kGvWarps) {
      const int nr = min(R, rc - rg * R);
      int a[R][MT][4];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int f = 0; f < 4; ++f) a[r][m][f] = 0;

      const uint8_t* wb = buf + (rg * R) * wstride;
      for (int c = lane; c < nchunk; c += 32) {
        uint32_t w[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          // chunks past the row's end read pad/other rows; their activations are zero
          uint4 v = make_uint4(0, 0, 0, 0);
          if (r < nr && c * 16 < wstride) v = *reinterpret_cast<const uint4*>(wb + r * wstride + c * 16);
          w[r][0] = v.x; w[r][1] = v.y; w[r][2] = v.z; w[r][3] = v.w;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const uint4* xp = reinterpret_cast<const uint4*>(xs + m * p.Kp + c * 64);
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint4 xv = xp[g];
#pragma unroll
            for (int r = 0; r < R; ++r) {
              const uint32_t wg = w[r][g];
              a[r][m][0] = dp4a_us(wg & 0x03030303u, xv.x, a[r][m][0]);
              a[r][m][1] = dp4a_us(wg & 0x0C0C0C0Cu, xv.y, a[r][m][1]);
              a[r][m][2] = dp4a_us(wg & 0x30303030u, xv.z, a[r][m][2]);
              a[r][m][3] = dp4a_us(wg & 0xC0C0C0C0u, xv.w, a[r][m][3]);
            }
          }
        }
      }
      // combine fields (exact: field f holds 4^f times its sum), reduce the warp
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          int t = a[r][m][0] + (a[r][m][1] >> 2) + (a[r][m][2] >> 4) + (a[r][m][3] >> 6);
          a[r][m][0] = warp_sum(t);
        }
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (lane == r * MT + m && r < nr && m < p.M) {
            const int64_t n = n0 + r0 + rg * R + r;
            int xsum = 0;
#pragma unroll
            for (int w = 0; w < kGvWarps; ++w) xsum += H.q.qpart[m][w];
            const int accv = a[r][m][0] - xsum;
            const int64_t idx = static_cast<int64_t>(m) * p.N + n;
            if (p.acc != nullptr) p.acc[idx] = accv;
            if (p.y != nullptr) store_y(p.y, p.y_dtype, idx, __fmul_rn(__int2float_rn(accv), __fmul_rn(gamma, H.scale[m])));
          }
        }
    }
    __syncthreads();
    if (p.bulk && tid == 0 && i + p.stages < nst) {
      fence_proxy_async_smem();
      issue(i + p.stages);
    }
  }
}

}  // namespace bitnet
