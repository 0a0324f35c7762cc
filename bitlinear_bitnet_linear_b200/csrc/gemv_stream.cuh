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
constexpr int kGsPrefetch = 12;    // weight stages pulled into L2 ahead of the ring

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
  int deep;                      // 1: long stream (tasks flow across stages), 0: one short call
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

// Short rows (M = 1, K <= 4096): a warp is four 8-lane groups, each owning
// RS consecutive rows; a lane walks every eighth code word of its rows, so a
// row's partial sums are reduced over 8 lanes (3 shuffles).  The groups start
// their walks 8 words apart (rotation modulo the row length), so rows whose
// word count is a multiple of 32 do not collide on shared-memory banks.
// Rows [row0, row0 + 4 RS) of the stage; requires nword % 8 == 0.
template <int RS>
__device__ __forceinline__ void gs_task_lanegroups(const uint32_t* wbase, int rc, int row0, int rowwords, int nword,
                                                   const int8_t* xs, int lane, int xsum0, float gs0,
                                                   const GsProblem& P, int r, int y_dtype) {
  const int lg = lane >> 3, lj = lane & 7;
  const int rb = row0 + lg * RS;                 // this group's first row
  const int nr = max(0, min(RS, rc - rb));
  int a[RS][4];
#pragma unroll
  for (int i = 0; i < RS; ++i)
#pragma unroll
    for (int f = 0; f < 4; ++f) a[i][f] = 0;
  const uint32_t* wb = wbase + static_cast<int64_t>(rb) * rowwords;
  int g = lj + 8 * lg;
  if (g >= nword) g -= nword * (g / nword);
  if (nr == RS) {
#pragma unroll 4
    for (int t = 0; t < nword; t += 8) {
      uint32_t w[RS];
#pragma unroll
      for (int i = 0; i < RS; ++i) w[i] = wb[i * rowwords + g];
      const uint4 xv = *reinterpret_cast<const uint4*>(xs + 16 * g);
#pragma unroll
      for (int i = 0; i < RS; ++i) {
        a[i][0] = dp4a_us(w[i] & 0x03030303u, xv.x, a[i][0]);
        a[i][1] = dp4a_us(w[i] & 0x0C0C0C0Cu, xv.y, a[i][1]);
        a[i][2] = dp4a_us(w[i] & 0x30303030u, xv.z, a[i][2]);
        a[i][3] = dp4a_us(w[i] & 0xC0C0C0C0u, xv.w, a[i][3]);
      }
      g += 8;
      if (g >= nword) g -= nword;
    }
  } else if (nr > 0) {
    for (int t = 0; t < nword; t += 8) {
      uint32_t w[RS];
#pragma unroll
      for (int i = 0; i < RS; ++i) w[i] = (i < nr) ? wb[i * rowwords + g] : 0u;
      const uint4 xv = *reinterpret_cast<const uint4*>(xs + 16 * g);
#pragma unroll
      for (int i = 0; i < RS; ++i) {
        a[i][0] = dp4a_us(w[i] & 0x03030303u, xv.x, a[i][0]);
        a[i][1] = dp4a_us(w[i] & 0x0C0C0C0Cu, xv.y, a[i][1]);
        a[i][2] = dp4a_us(w[i] & 0x30303030u, xv.z, a[i][2]);
        a[i][3] = dp4a_us(w[i] & 0xC0C0C0C0u, xv.w, a[i][3]);
      }
      g += 8;
      if (g >= nword) g -= nword;
    }
  }
#pragma unroll
  for (int i = 0; i < RS; ++i) {
    int t = a[i][0] + (a[i][1] >> 2) + (a[i][2] >> 4) + (a[i][3] >> 6);
    t += __shfl_xor_sync(0xffffffffu, t, 4);
    t += __shfl_xor_sync(0xffffffffu, t, 2);
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    a[i][0] = t;
  }
#pragma unroll
  for (int i = 0; i < RS; ++i) {
    if (lj == i && i < nr) {
      const int64_t n = r + rb + i;
      const int accv = a[i][0] - xsum0;
      if (P.acc != nullptr) P.acc[n] = accv;
      if (P.y != nullptr) store_y(P.y, y_dtype, n, __fmul_rn(__int2float_rn(accv), gs0));
    }
  }
}

// Long rows or M > 1: a warp owns R rows, lane l walks code words l, l + 32, ...
// Rows [row0, row0 + R) of the stage.
template <int R, int MT>
__device__ __forceinline__ void gs_task_warp(const uint32_t* wbase, int rc, int row0, int rowwords, int nword,
                                             const int8_t* xs, int Kp, int lane, const int (&xsum)[MT],
                                             const float (&sc)[MT], float gamma, const GsProblem& P, int r, int M,
                                             int y_dtype) {
  const int nr = min(R, rc - row0);
  int a[R][MT][4];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
      for (int f = 0; f < 4; ++f) a[i][m][f] = 0;
  const uint32_t* wb = wbase + static_cast<int64_t>(row0) * rowwords;
  auto body = [&](const uint32_t (&w)[R], int g) {
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
  };
  if (nr == R) {
#pragma unroll 4
    for (int g = lane; g < nword; g += 32) {
      uint32_t w[R];
#pragma unroll
      for (int i = 0; i < R; ++i) w[i] = wb[i * rowwords + g];
      body(w, g);
    }
  } else {
    for (int g = lane; g < nword; g += 32) {
      uint32_t w[R];
#pragma unroll
      for (int i = 0; i < R; ++i) w[i] = (i < nr) ? wb[i * rowwords + g] : 0u;
      body(w, g);
    }
  }
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
        const int64_t n = r + row0 + i;
        const int accv = a[i][m][0] - xsum[m];
        const int64_t idx = static_cast<int64_t>(m) * P.N + n;
        if (P.acc != nullptr) P.acc[idx] = accv;
        if (P.y != nullptr) store_y(P.y, y_dtype, idx, __fmul_rn(__int2float_rn(accv), __fmul_rn(gamma, sc[m])));
      }
    }
}

// CW consumer warps + one producer warp.
template <int MT, int MAXP, int CW, bool DEEP>
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
      // L2 prefetch cursor: walks the same stage sequence kGsPrefetch stages
      // ahead of the shared-memory copies, so those copies hit in L2 and the
      // DRAM stream does not wait for ring slots to be released.
      int pq = pb, pr = (pb <= qlast) ? rb : 0, npf = 0;
      auto prefetch_upto = [&](int upto) {
        while (npf < upto && pq <= qlast) {
          int q0, q1;
          seg_bounds(pq, q0, q1);
          if (pr >= q1) {
            ++pq;
            if (pq <= qlast) seg_bounds(pq, pr, q1);
            continue;
          }
          const GsProblem& Q = p.prob[pq];
          const int64_t qrowb = Q.K / 4;
          const int rc = min(Q.srows, q1 - pr);
          bulk_prefetch_l2(Q.Wp + static_cast<int64_t>(pr) * qrowb, static_cast<uint32_t>(rc * qrowb));
          pr += Q.srows;
          ++npf;
        }
      };
      prefetch_upto(kGsPrefetch);
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
            prefetch_upto(issued + kGsPrefetch);
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
          prefetch_upto(t + kGsPrefetch);
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
  int64_t task0 = 0;
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
    // Work units ("tasks") of every stage are numbered globally and dealt to
    // the warps round-robin, so a warp with nothing to do in one stage moves
    // on to the next; a slot is released when every warp has passed it.
    const bool lanegroups = (MT == 1) && (P.K <= 4096) && (nword % 8 == 0);
    const float gs0 = __fmul_rn(gamma, sc[0]);
    for (int r = r0; r < r1; r += P.srows, ++ts) {
      const int s = ts % p.nslots;
      const int rc = min(P.srows, r1 - r);
      // task size for this stage (identical in every warp): the largest that
      // still gives every warp work, up to 16 rows (4 per 8-lane group) or 4
      // rows per warp
      int kind, rows_per_task;
      if constexpr (DEEP) {
        // long streams: fixed task sizes (8-row lane-group tasks; 4/2/1-row
        // warp tasks by M); stages hold one task per warp
        kind = lanegroups ? 2 : (MT == 1 ? 4 : (MT == 2 ? 2 : 1));
        rows_per_task = lanegroups ? 4 * kind : kind;
      } else if (lanegroups) {
        kind = ((rc + 15) / 16 >= kGsWarps) ? 4 : 1;
        rows_per_task = 4 * kind;
      } else {
        auto cost = [&](int RR) { return ((rc + RR - 1) / RR + kGsWarps - 1) / kGsWarps * RR; };
        kind = 1;
        if (MT <= 2 && cost(2) <= cost(1)) kind = 2;
        if (MT == 1 && cost(4) <= cost(kind)) kind = 4;
        rows_per_task = kind;
      }
      const int nt = (rc + rows_per_task - 1) / rows_per_task;
      const int j0 = (warp - static_cast<int>(task0 % kGsWarps) + kGsWarps) % kGsWarps;
      // Every warp waits for every stage to land, even one with no task in
      // it, before releasing it: a warp is then never more than one phase of
      // a slot ahead of the others, which keeps the parity waits and the
      // release counts of each slot's barriers exact.
      const bool got = mbar_wait_bounded(&H.wfull[s], (ts / p.nslots) & 1, p.limit_ns, abort_flag);
      if (!got && !*abort_flag) {
        record_error(p.status, BITNET_ERR_TIMEOUT, 0x403u);
        *abort_flag = 1;
      }
      if (j0 < nt) {
        if (got) {
          const uint32_t* wbase = reinterpret_cast<const uint32_t*>(wring + s * p.slot_bytes);
          for (int j = j0; j < nt; j += kGsWarps) {
            const int row0 = j * rows_per_task;
            if (lanegroups) {
              if constexpr (DEEP) {
                gs_task_lanegroups<2>(wbase, rc, row0, rowwords, nword, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
              } else {
                if (kind == 4)
                  gs_task_lanegroups<4>(wbase, rc, row0, rowwords, nword, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
                else
                  gs_task_lanegroups<1>(wbase, rc, row0, rowwords, nword, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
              }
            } else if constexpr (DEEP) {
              gs_task_warp<(MT == 1 ? 4 : (MT == 2 ? 2 : 1)), MT>(wbase, rc, row0, rowwords, nword, xs, Kp, lane, xsum,
                                                                   sc, gamma, P, r, p.M, p.y_dtype);
            } else if (kind == 4) {
              if constexpr (MT == 1)
                gs_task_warp<4, MT>(wbase, rc, row0, rowwords, nword, xs, Kp, lane, xsum, sc, gamma, P, r, p.M,
                                    p.y_dtype);
            } else if (kind == 2) {
              if constexpr (MT <= 2)
                gs_task_warp<2, MT>(wbase, rc, row0, rowwords, nword, xs, Kp, lane, xsum, sc, gamma, P, r, p.M,
                                    p.y_dtype);
            } else {
              gs_task_warp<1, MT>(wbase, rc, row0, rowwords, nword, xs, Kp, lane, xsum, sc, gamma, P, r, p.M,
                                  p.y_dtype);
            }
          }
        }
      }
      task0 += nt;
      __syncwarp();
      if (lane == 0) mbar_arrive(&H.wempty[s]);
    }
  }
  if (!triggered) pdl_launch_dependents();
}

}  // namespace bitnet
