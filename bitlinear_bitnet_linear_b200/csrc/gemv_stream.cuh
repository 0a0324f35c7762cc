// gemv_stream.cuh -- packed-ternary GEMV over one or many problems (decode).
//
// For each problem p:  y_p[m,n] = (sum_k x_q[m,k] W_q[n,k]) * gamma_p * s_x[m]
// with M <= 4 tokens.  The ternary dot product ("sum of activations where
// the weight is +1 minus the sum where it is -1", Hacker News thread on the
// b1.58 paper) is formed from the stored codes c = q + 1:
//     sum_k q_k x_k = sum_k c_k x_k - sum_k x_k,
// masking field s of a packed 32-bit group (0x03030303 << 2s) lines four
// codes (scaled by 4^s) up with four consecutive int8 activations for
// dp4a; four per-field accumulators are rescaled by exact shifts.
//
// One launch streams the packed weights of every problem it is given.  The
// concatenated weight bytes are split evenly over the CTAs; each CTA walks
// its range as segments (problem, row range).  Roles:
//   warp 8      producer: cp.async.bulk (TMA, no multicast) of weight stages
//               into a ring of shared-memory slots and of each segment's raw
//               activation rows into a small ring, tracked by mbarriers;
//               weight stages are issued before griddepcontrol.wait (weights
//               never depend on earlier kernels), activations after it.
//   warps 0..7  consumers: quantise a segment's activations from shared
//               memory (fused RMSNorm gain + absmax int8, skipped when the
//               segment shares the previous one's activations), then
//               contract every stage's rows, reduce across lanes and write y.
// Problems that share x (fused Q|K|V, up|gate) are quantised once per CTA.
// Every wait is bounded: on expiry the kernel records BITNET_ERR_TIMEOUT,
// stops issuing, lets copies already issued land, and returns.
#pragma once

#include "act.cuh"
#include "common.cuh"

namespace bitnet {

constexpr int kGsMaxSlots = 12;
constexpr int kGsMaxX = 2;
constexpr int kGsHeader = 2048;
constexpr int kGsBar = 1;          // named barrier of the consumer warps

struct GsProblem {
  const void* x;          // [M, K] raw activations (x_dtype) or int8 codes (prequant)
  const uint8_t* Wp;      // [N, K/4]
  const float* gamma;     // device scalar
  const float* gain;      // [K] RMSNorm gain or nullptr
  const float* x_scale;   // [M] (prequant only)
  void* y;                // [M, N] or nullptr
  int32_t* acc;           // [M, N] exact accumulator export or nullptr
  int K, N;
  int srows;              // rows per weight stage
  int pad;
  int64_t byte0;          // first byte of this problem in the concatenated weight stream
};

template <int MAXP>
struct GsParams {
  GsProblem prob[MAXP];
  int nprob;
  int M, x_dtype, y_dtype, prequant;
  float rms_eps;
  int64_t total_bytes;
  int slot_bytes, nslots;        // weight ring
  int xbuf_bytes, nxbuf;         // activation ring (nxbuf == 0: read x from global memory)
  int Kp_max;                    // int8 code rows in shared memory, K rounded up to 64
  uint64_t limit_ns;
  uint32_t* status;
};

template <int MT, int CW>
struct GsHeader {
  uint64_t wfull[kGsMaxSlots], wempty[kGsMaxSlots];
  uint64_t xfull[kGsMaxX], xempty[kGsMaxX];
  QuantScratch<CW * 32, MT> q;
  int abort;
};

// First global row (problem, row) of CTA b's share of the weight bytes.
template <int MAXP>
__device__ __forceinline__ void gs_cta_start(const GsParams<MAXP>& p, int b, int& prob, int& row) {
  const int64_t target = (p.total_bytes * b) / gridDim.x;
  for (int i = 0; i < p.nprob; ++i) {
    const int64_t rb = p.prob[i].K / 4;
    const int64_t end = p.prob[i].byte0 + rb * p.prob[i].N;
    if (target < end) {
      const int64_t r = (target - p.prob[i].byte0 + rb - 1) / rb;
      if (r < p.prob[i].N) {
        prob = i;
        row = static_cast<int>(r);
        return;
      }
    }
  }
  prob = p.nprob;
  row = 0;
}

// Contract the rows of one weight stage (rc rows starting at problem row r)
// against the shared-memory activation codes; warps take groups of R rows,
// lane l takes code words l, l + 32, ... of those rows.
template <int R, int MT, int CW>
__device__ __forceinline__ void gs_contract(const uint8_t* buf, int rc, int rowwords, int nword, const int8_t* xs,
                                            int Kp, int warp, int lane, const int (&xsum)[MT],
                                            const float (&sc)[MT], float gamma, const GsProblem& P, int r, int M,
                                            int y_dtype) {
  for (int rg = warp; rg * R < rc; rg += CW) {
    const int nr = min(R, rc - rg * R);
    int a[R][MT][4];
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int f = 0; f < 4; ++f) a[i][m][f] = 0;
    const uint32_t* wb = reinterpret_cast<const uint32_t*>(buf) + (rg * R) * rowwords;
    // 16 weights (one code word) against the 16 activations at bytes [16 g, 16 g + 16)
#pragma unroll 2
    for (int g = lane; g < nword; g += 32) {
      uint32_t w[R];
#pragma unroll
      for (int i = 0; i < R; ++i) w[i] = (i < nr) ? wb[i * rowwords + g] : 0u;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xs + m * Kp + 16 * g);
#pragma unroll
        for (int i = 0; i < R; ++i) {
          a[i][m][0] = dp4a_us(w[i] & 0x03030303u, xv.x, a[i][m][0]);
          a[i][m][1] = dp4a_us(w[i] & 0x0C0C0C0Cu, xv.y, a[i][m][1]);
          a[i][m][2] = dp4a_us(w[i] & 0x30303030u, xv.z, a[i][m][2]);
          a[i][m][3] = dp4a_us(w[i] & 0xC0C0C0C0u, xv.w, a[i][m][3]);
        }
      }
    }
    // field f holds 4^f times its sum: exact shifts, then the lane reduction
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int m = 0; m < MT; ++m)
        a[i][m][0] = warp_sum(a[i][m][0] + (a[i][m][1] >> 2) + (a[i][m][2] >> 4) + (a[i][m][3] >> 6));
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (lane == i * MT + m && i < nr && m < M) {
          const int64_t n = r + rg * R + i;
          const int accv = a[i][m][0] - xsum[m];
          const int64_t idx = static_cast<int64_t>(m) * P.N + n;
          if (P.acc != nullptr) P.acc[idx] = accv;
          if (P.y != nullptr) store_y(P.y, y_dtype, idx, __fmul_rn(__int2float_rn(accv), __fmul_rn(gamma, sc[m])));
        }
      }
  }
}

// CW consumer warps + one producer warp.
template <int MT, int MAXP, int CW>
__global__ void __launch_bounds__(CW * 32 + 32, (CW <= 8 ? 2 : 1))
    gemv_stream_kernel(const __grid_constant__ GsParams<MAXP> p) {
  constexpr int kGsConsumers = CW * 32;
  constexpr int kGsWarps = CW;
  extern __shared__ __align__(128) uint8_t smem[];
  static_assert(sizeof(GsHeader<MT, CW>) <= kGsHeader, "header too large");
  GsHeader<MT, CW>& H = *reinterpret_cast<GsHeader<MT, CW>*>(smem);
  int8_t* xs = reinterpret_cast<int8_t*>(smem + kGsHeader);
  uint8_t* xraw = smem + kGsHeader + MT * p.Kp_max;
  uint8_t* wring = xraw + p.nxbuf * p.xbuf_bytes;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int pb, rb, pe, re;
  gs_cta_start(p, blockIdx.x, pb, rb);
  gs_cta_start(p, blockIdx.x + 1, pe, re);
  if (blockIdx.x + 1 == gridDim.x) {
    pe = p.nprob;
    re = 0;
  }
  // segment iteration: problem q from pb to pe (inclusive when re > 0)
  auto seg_bounds = [&](int q, int& r0, int& r1) {
    r0 = (q == pb) ? rb : 0;
    r1 = (q == pe) ? re : p.prob[q].N;
  };
  const int qlast = (re > 0) ? pe : pe - 1;
  auto shares_x = [&](int q) {   // segment q reuses segment q-1's quantised activations
    return q > pb && p.prob[q].x == p.prob[q - 1].x && p.prob[q].gain == p.prob[q - 1].gain &&
           p.prob[q].K == p.prob[q - 1].K && p.prob[q].x_scale == p.prob[q - 1].x_scale;
  };
  const int64_t esz = p.prequant ? 1 : (p.x_dtype == BITNET_BF16 ? 2 : 4);

  if (tid == 0) {
    for (int s = 0; s < p.nslots; ++s) {
      mbar_init(&H.wfull[s], 1);
      mbar_init(&H.wempty[s], kGsWarps);
    }
    for (int s = 0; s < p.nxbuf; ++s) {
      mbar_init(&H.xfull[s], 1);
      mbar_init(&H.xempty[s], kGsWarps);
    }
    H.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &H.abort;

  if (warp == kGsWarps) {
    // ================================================================ producer
    if (lane != 0) {
      pdl_launch_dependents();
      return;
    }
    {
      int t = 0;          // weight stages issued
      int u = 0;          // activation buffers issued
      bool dep_waited = false;
      bool ok = true;
      // Phase 1: fill the weight ring before the dependency wait.
      {
        int issued = 0;
        for (int q = pb; q <= qlast && issued < p.nslots; ++q) {
          int r0, r1;
          seg_bounds(q, r0, r1);
          const GsProblem& P = p.prob[q];
          const int64_t rowb = P.K / 4;
          for (int r = r0; r < r1 && issued < p.nslots; r += P.srows) {
            const int rc = min(P.srows, r1 - r);
            const uint32_t bytes = static_cast<uint32_t>(rc * rowb);
            mbar_expect_tx(&H.wfull[issued], bytes);
            bulk_g2s(wring + issued * p.slot_bytes, P.Wp + static_cast<int64_t>(r) * rowb, bytes, &H.wfull[issued]);
            ++issued;
          }
        }
        t = issued;
      }
      // Phase 2: activations (after the dependency wait) and the rest of the weights.
      int ts = 0;   // global stage index while walking
      for (int q = pb; q <= qlast && ok; ++q) {
        int r0, r1;
        seg_bounds(q, r0, r1);
        const GsProblem& P = p.prob[q];
        if (!shares_x(q)) {
          if (!dep_waited) {
            pdl_wait();
            pdl_launch_dependents();
            dep_waited = true;
          }
          if (p.nxbuf > 0) {
            const int xi = u % p.nxbuf;
            if (!mbar_wait_bounded(&H.xempty[xi], ((u / p.nxbuf) & 1) ^ 1u, p.limit_ns, abort_flag)) {
              ok = false;
              break;
            }
            const uint32_t bytes = static_cast<uint32_t>(p.M * P.K * esz);
            mbar_expect_tx(&H.xfull[xi], bytes);
            bulk_g2s(xraw + xi * p.xbuf_bytes, P.x, bytes, &H.xfull[xi]);
          }
          ++u;
        }
        const int64_t rowb = P.K / 4;
        for (int r = r0; r < r1; r += P.srows, ++ts) {
          if (ts < t) continue;   // issued in phase 1
          const int s = ts % p.nslots;
          if (!mbar_wait_bounded(&H.wempty[s], ((ts / p.nslots) & 1) ^ 1u, p.limit_ns, abort_flag)) {
            ok = false;
            break;
          }
          const int rc = min(P.srows, r1 - r);
          const uint32_t bytes = static_cast<uint32_t>(rc * rowb);
          mbar_expect_tx(&H.wfull[s], bytes);
          bulk_g2s(wring + s * p.slot_bytes, P.Wp + static_cast<int64_t>(r) * rowb, bytes, &H.wfull[s]);
          ++t;
        }
      }
      if (!dep_waited) {
        pdl_wait();
        pdl_launch_dependents();
      }
      if (!ok) {
        if (!*abort_flag) {
          record_error(p.status, BITNET_ERR_TIMEOUT, 0x401u);
          *abort_flag = 1;
        }
        // let every weight copy still in flight land before the CTA exits
        for (int i = max(0, t - p.nslots); i < t; ++i)
          mbar_wait_bounded(&H.wfull[i % p.nslots], (i / p.nslots) & 1, p.limit_ns, nullptr);
        for (int i = max(0, u - p.nxbuf); i < u && p.nxbuf > 0; ++i)
          mbar_wait_bounded(&H.xfull[i % p.nxbuf], (i / p.nxbuf) & 1, p.limit_ns, nullptr);
      }
    }
    return;
  }

  // ================================================================== consumers
  float sc[MT];
  int xsum[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    sc[m] = 0.0f;
    xsum[m] = 0;
  }
  int ts = 0, u = 0;
  bool triggered = false;
  for (int q = pb; q <= qlast; ++q) {
    int r0, r1;
    seg_bounds(q, r0, r1);
    const GsProblem& P = p.prob[q];
    const int Kp = (P.K + 63) & ~63;
    if (!shares_x(q)) {
      // all consumers are done with the previous segment's codes
      group_sync<kGsBar, kGsConsumers>();
      bool have = true;
      const char* src = static_cast<const char*>(P.x);
      if (p.nxbuf > 0) {
        const int xi = u % p.nxbuf;
        have = mbar_wait_bounded(&H.xfull[xi], (u / p.nxbuf) & 1, p.limit_ns, abort_flag);
        src = reinterpret_cast<const char*>(xraw + xi * p.xbuf_bytes);
      } else {
        pdl_wait();
      }
      if (!have && !*abort_flag) {
        record_error(p.status, BITNET_ERR_TIMEOUT, 0x402u);
        *abort_flag = 1;
      }
      const bool live = !*abort_flag;
      if (p.prequant) {
        // copy codes (swizzled) and form their sums
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          int part = 0;
          if (live && m < p.M) {
            for (int k = tid * 16; k < P.K; k += kGsConsumers * 16) {
              const uint4 v = p.nxbuf > 0 ? *reinterpret_cast<const uint4*>(src + m * P.K + k)
                                          : __ldg(reinterpret_cast<const uint4*>(src + m * P.K + k));
              *reinterpret_cast<uint4*>(xs + m * Kp + k) = v;
              part = __dp4a(static_cast<int>(v.x), 0x01010101, part);
              part = __dp4a(static_cast<int>(v.y), 0x01010101, part);
              part = __dp4a(static_cast<int>(v.z), 0x01010101, part);
              part = __dp4a(static_cast<int>(v.w), 0x01010101, part);
            }
          }
          part = warp_sum(part);
          if (lane == 0) H.q.qpart[m][warp] = part;
          sc[m] = (live && m < p.M) ? __ldg(P.x_scale + m) : 0.0f;
        }
      } else if (live) {
        if (p.nxbuf > 0)
          quant_rows<kGsConsumers, MT, (MT == 1 ? 2 : 1), true, kGsBar, false>(
              src, p.x_dtype, P.K * esz, p.M, P.K, P.gain, p.rms_eps, xs, Kp, H.q, sc);
        else
          quant_rows<kGsConsumers, MT, (MT == 1 ? 2 : 1), false, kGsBar, false>(
              src, p.x_dtype, P.K * esz, p.M, P.K, P.gain, p.rms_eps, xs, Kp, H.q, sc);
      } else {
        group_sync<kGsBar, kGsConsumers>();   // the barrier inside quant_rows
      }
      // zero padding: codes past K (within the last 64-wide chunk) and rows past M
      for (int m = 0; m < MT; ++m) {
        const int k0 = (m < p.M) ? P.K : 0;
        for (int k = k0 + tid * 16; k < Kp; k += kGsConsumers * 16)
          *reinterpret_cast<uint4*>(xs + m * Kp + k) = make_uint4(0, 0, 0, 0);
      }
      group_sync<kGsBar, kGsConsumers>();
      if (p.nxbuf > 0 && lane == 0) mbar_arrive(&H.xempty[u % p.nxbuf]);
      ++u;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        int t = 0;
#pragma unroll
        for (int w = 0; w < kGsWarps; ++w) t += H.q.qpart[m][w];
        xsum[m] = t;
      }
      if (!triggered) {
        pdl_launch_dependents();
        triggered = true;
      }
    }

    const float gamma = __ldg(P.gamma);
    const int64_t rowb = P.K / 4;
    const int nword = P.K / 16;      // 32-bit code words (16 weights) per row
    const int rowwords = static_cast<int>(rowb / 4);
    for (int r = r0; r < r1; r += P.srows, ++ts) {
      const int s = ts % p.nslots;
      const bool got = mbar_wait_bounded(&H.wfull[s], (ts / p.nslots) & 1, p.limit_ns, abort_flag);
      if (!got && !*abort_flag) {
        record_error(p.status, BITNET_ERR_TIMEOUT, 0x403u);
        *abort_flag = 1;
      }
      const int rc = min(P.srows, r1 - r);
      const uint8_t* buf = wring + s * p.slot_bytes;
      if (got) {
        // rows per warp task: the smallest critical path (rounds of warp
        // tasks x rows per task), ties to the larger task, which reuses each
        // activation word across more rows
        auto cost = [&](int RR) { return ((rc + RR - 1) / RR + CW - 1) / CW * RR; };
        if constexpr (MT == 1) {
          const int c1 = cost(1), c2 = cost(2), c4 = cost(4);
          if (c4 <= c2 && c4 <= c1)
            gs_contract<4, MT, CW>(buf, rc, rowwords, nword, xs, Kp, warp, lane, xsum, sc, gamma, P, r, p.M, p.y_dtype);
          else if (c2 <= c1)
            gs_contract<2, MT, CW>(buf, rc, rowwords, nword, xs, Kp, warp, lane, xsum, sc, gamma, P, r, p.M, p.y_dtype);
          else
            gs_contract<1, MT, CW>(buf, rc, rowwords, nword, xs, Kp, warp, lane, xsum, sc, gamma, P, r, p.M, p.y_dtype);
        } else if constexpr (MT == 2) {
          if (cost(2) <= cost(1))
            gs_contract<2, MT, CW>(buf, rc, rowwords, nword, xs, Kp, warp, lane, xsum, sc, gamma, P, r, p.M, p.y_dtype);
          else
            gs_contract<1, MT, CW>(buf, rc, rowwords, nword, xs, Kp, warp, lane, xsum, sc, gamma, P, r, p.M, p.y_dtype);
        } else {
          gs_contract<1, MT, CW>(buf, rc, rowwords, nword, xs, Kp, warp, lane, xsum, sc, gamma, P, r, p.M, p.y_dtype);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&H.wempty[s]);
    }
  }
  if (!triggered) pdl_launch_dependents();
}

}  // namespace bitnet
