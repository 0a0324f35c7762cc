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
// its range as segments (problem, row range), and cuts every segment into
// chunks of whole rows that fit one shared-memory slot.  Roles:
//   warps 0..CW-1  consumers.  Chunk j of the CTA belongs to warp j % CW.
//                  Each consumer keeps its own ring of slots: its lane 0
//                  issues cp.async.bulk (TMA, no multicast) of its next
//                  chunks into them, so no consumer ever waits for another
//                  to release a slot.  The first copies go out before
//                  griddepcontrol.wait (weights never depend on earlier
//                  kernels).
//   warp CW        activations.  Quantises each segment's activations
//                  (fused RMSNorm gain + absmax int8, skipped when a segment
//                  shares the previous one's activations) one segment ahead
//                  of the consumers, into two alternating buffers (one
//                  when long rows leave no room: then it waits for the
//                  consumers to finish a segment before quantising the next).
//                  The first segment is quantised by every warp together.
// Four warps per scheduler hide the latency of the 128-bit shared loads and
// of the dp4a chains.  Every wait is bounded: on expiry the kernel records
// BITNET_ERR_TIMEOUT, stops issuing, lets copies already issued land, and
// returns.
#pragma once

#include "act.cuh"
#include "common.cuh"

namespace bitnet {

constexpr int kGsMaxS = 4;          // slots per consumer warp
constexpr int kGsCW = 15;           // consumer warps per CTA
constexpr int kGsHeader = 2048;
constexpr int kGsBarAll = 1;        // named barrier: every warp of the CTA
constexpr int kGsBarX = 2;          // named barrier: the activation warp

// Consumer task shapes (per problem): lane groups of G lanes with RS rows
// each (M = 1, block-permuted codes), or whole warps.
constexpr int kGsTaskG8R2 = 0;      // 8-row tasks
constexpr int kGsTaskG16R2 = 1;     // 4-row tasks
constexpr int kGsTaskG16R1 = 2;     // 2-row tasks
constexpr int kGsTaskG32R1 = 3;     // 1-row tasks
constexpr int kGsTaskWarp = 4;      // whole warp over R = 4 / 2 / 1 rows (M = 1 / 2 / 4), linear codes
constexpr int kGsTaskB1 = 5;        // 1-bit signs: kGsTaskB1 + (a G/RS shape above, 0 .. 3)
constexpr int kGsTaskT3 = 9;        // base-3: whole warp over 4 rows, linear codes

struct GsProblem {
  const void* x;          // [M, K] raw activations (x_dtype) or int8 codes (prequant)
  const void* x2;         // [M, K] up projection for a ReLU^2-gated input (x is the gate), or nullptr
  const void* resid;      // [M, N] residual added to y (y_dtype), or nullptr
  const uint8_t* Wp;      // [N, K/4]
  const float* gamma;     // device scalar
  const float* gain;      // [K] RMSNorm gain or nullptr
  const float* x_scale;   // [M] (prequant only)
  void* y;                // [M, N] or nullptr
  int32_t* acc;           // [M, N] exact accumulator export or nullptr
  int K, N;
  int rc;                 // rows per chunk (one slot)
  int task;               // kGsTask*
  int64_t byte0;          // first byte of this problem in the concatenated weight stream
};

template <int MAXP>
struct GsParams {
  GsProblem prob[MAXP];
  int nprob;
  int M, x_dtype, y_dtype, prequant;
  float rms_eps;
  int64_t total_bytes;
  int slot_bytes, nslots;        // ring of each consumer warp
  int nxb;                       // activation code buffers (2: quantise a segment ahead)
  int blocked;                   // 1 / 2: codes block-permuted in 4 / 8 quarters (lane-group tasks)
  int bits;                      // 2: ternary codes, 2 bits per weight; 1: BitNet b1 signs; 3: base-3
  int Kp_max;                    // int8 code rows in shared memory (K rounded up to 64)
  uint64_t limit_ns;
  uint32_t* status;
};

template <int MT, int CW>
struct GsHeader {
  uint64_t wfull[CW][kGsMaxS];
  uint64_t xfull[2], xfree[2], xcopy;   // xcopy: pre-quantised codes copied in
  float scale[2][MT];
  int xsum[2][MT];
  QuantScratch<(CW + 1) * 32, MT> q;   // first segment (every warp)
  QuantScratch<32, MT> qx;             // later segments (activation warp)
  int abort;
};

// Bytes of one packed row and the code-row length in shared memory, by
// weight format: bits 2 (ternary codes, K/4 bytes), 1 (BitNet b1 signs,
// K/8 bytes) or 3 (base-3, five weights per byte, ceil(K/80) 16-byte chunks;
// the code row is zero-padded to a multiple of 80).
__host__ __device__ __forceinline__ int64_t gs_row_bytes(int64_t K, int bits) {
  return bits == 3 ? (K + 79) / 80 * 16 : K / 8 * bits;
}
__host__ __device__ __forceinline__ int gs_code_row(int K, int bits) {
  return bits == 3 ? (K + 79) / 80 * 80 : (K + 63) & ~63;
}

// First global row (problem, row) of CTA b's share of the weight bytes: the
// first row that starts at or after byte total * b / gridDim.x (binary
// search over the problems' byte ranges).
template <int MAXP>
__device__ __forceinline__ void gs_cta_start(const GsParams<MAXP>& p, int b, int& prob, int& row) {
  const int64_t target = (p.total_bytes * b) / gridDim.x;
  int lo = 0, hi = p.nprob;   // first problem whose bytes end after target
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int64_t end = p.prob[mid].byte0 + gs_row_bytes(p.prob[mid].K, p.bits) * p.prob[mid].N;
    if (target < end)
      hi = mid;
    else
      lo = mid + 1;
  }
  prob = lo;
  row = 0;
  if (lo == p.nprob) return;
  const int64_t rb = gs_row_bytes(p.prob[lo].K, p.bits);
  // target may sit inside the previous problem's last row (before byte0)
  const int64_t off = target > p.prob[lo].byte0 ? target - p.prob[lo].byte0 : 0;
  const int64_t r = (off + rb - 1) / rb;
  if (r < p.prob[lo].N)
    row = static_cast<int>(r);
  else
    prob = lo + 1;            // inside the last row of problem lo: the next one starts at row 0
}

// A chunk position: rows [r, min(r + rc, r1)) of problem q.
struct GsCursor {
  int q, r, r1;
};

// Warp-uniform bounded wait: true only when every lane saw the phase complete.
__device__ __forceinline__ bool gs_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                        volatile int* abort_flag) {
  return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, limit_ns, abort_flag));
}

// M = 1: a warp is 32/G groups of G lanes (G = 8, 16 or 32), each owning RS
// consecutive rows of the chunk.  A lane reads 16 bytes of packed codes per
// row at a time (64 weights, chunk c = lj, lj + G, ...) and the four 16-byte
// activation blocks they meet from the block-permuted code row (xs_blocked),
// all with 128-bit shared loads; every 8 consecutive lanes read 128
// consecutive bytes, so no load has a bank conflict.  A row's partial sums
// are reduced over its G lanes.  Rows [row0, row0 + (32/G) RS) of the chunk.
template <int G, int RS>
__device__ __forceinline__ void gs_task_lg(const uint8_t* wbase, int rc, int row0, int rowb, int nchunk,
                                           const int8_t* xs, int lane, int xsum0, float gs0, const GsProblem& P,
                                           int r, int y_dtype) {
  const int lg = lane / G, lj = lane % G;
  const int rb = row0 + lg * RS;                 // this group's first row
  const int nr = max(0, min(RS, rc - rb));
  const int xq4 = rowb;                          // K / 4: distance between the four block quarters
  int a[RS][4];
#pragma unroll
  for (int i = 0; i < RS; ++i)
#pragma unroll
    for (int f = 0; f < 4; ++f) a[i][f] = 0;
  auto body = [&](const uint4 (&w)[RS], const int8_t* xp) {
    const uint4 xv[4] = {*reinterpret_cast<const uint4*>(xp), *reinterpret_cast<const uint4*>(xp + xq4),
                         *reinterpret_cast<const uint4*>(xp + 2 * xq4),
                         *reinterpret_cast<const uint4*>(xp + 3 * xq4)};
#pragma unroll
    for (int i = 0; i < RS; ++i) {
      const uint32_t wv[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        a[i][0] = dp4a_us(wv[e] & 0x03030303u, xv[e].x, a[i][0]);
        a[i][1] = dp4a_us(wv[e] & 0x0C0C0C0Cu, xv[e].y, a[i][1]);
        a[i][2] = dp4a_us(wv[e] & 0x30303030u, xv[e].z, a[i][2]);
        a[i][3] = dp4a_us(wv[e] & 0xC0C0C0C0u, xv[e].w, a[i][3]);
      }
    }
  };
  const uint8_t* wrow = wbase + static_cast<int64_t>(rb) * rowb + 16 * lj;
  const int8_t* xp = xs + 16 * lj;
  if (nr == RS) {
#pragma unroll 2
    for (int c = lj; c < nchunk; c += G) {
      uint4 w[RS];
#pragma unroll
      for (int i = 0; i < RS; ++i) w[i] = *reinterpret_cast<const uint4*>(wrow + i * rowb);
      body(w, xp);
      wrow += 16 * G;
      xp += 16 * G;
    }
  } else if (nr > 0) {
    for (int c = lj; c < nchunk; c += G) {
      uint4 w[RS];
#pragma unroll
      for (int i = 0; i < RS; ++i)
        w[i] = (i < nr) ? *reinterpret_cast<const uint4*>(wrow + i * rowb) : make_uint4(0u, 0u, 0u, 0u);
      body(w, xp);
      wrow += 16 * G;
      xp += 16 * G;
    }
  }
#pragma unroll
  for (int i = 0; i < RS; ++i) {
    int t = a[i][0] + (a[i][1] >> 2) + (a[i][2] >> 4) + (a[i][3] >> 6);
#pragma unroll
    for (int o = G / 2; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    a[i][0] = t;
  }
#pragma unroll
  for (int i = 0; i < RS; ++i) {
    if (lj == i && i < nr) {
      const int64_t n = r + rb + i;
      const int accv = a[i][0] - xsum0;
      if (P.acc != nullptr) P.acc[n] = accv;
      if (P.y != nullptr) {
        float o = __fmul_rn(__int2float_rn(accv), gs0);
        if (P.resid != nullptr) o = __fadd_rn(load_y(P.resid, y_dtype, n), o);
        store_y(P.y, y_dtype, n, o);
      }
    }
  }
}

// BitNet b1 signs, M = 1: as gs_task_lg, with 16 bytes of packed signs per
// row per step (128 weights, chunk c) against eight 16-byte activation
// blocks (xs_blocked8).  Word e of the chunk holds weights 32e + 4s + j at
// bit 8j + s; masking field s (0x01010101 << s) lines four signs (scaled by
// 2^s) up with four activations; eight per-field accumulators are rescaled
// by exact shifts.  With signs b = (q + 1) / 2: sum q x = 2 sum b x - sum x.
template <int G, int RS>
__device__ __forceinline__ void gs_task_lg_b1(const uint8_t* wbase, int rc, int row0, int rowb, int nchunk,
                                              const int8_t* xs, int lane, int xsum0, float gs0, const GsProblem& P,
                                              int r, int y_dtype) {
  const int lg = lane / G, lj = lane % G;
  const int rb = row0 + lg * RS;
  const int nr = max(0, min(RS, rc - rb));
  const int xq8 = rowb;                          // K / 8: distance between the eight block quarters
  int a[RS][8];
#pragma unroll
  for (int i = 0; i < RS; ++i)
#pragma unroll
    for (int f = 0; f < 8; ++f) a[i][f] = 0;
  auto body = [&](const uint4 (&w)[RS], const int8_t* xp) {
    uint4 xv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) xv[e] = *reinterpret_cast<const uint4*>(xp + e * xq8);
#pragma unroll
    for (int i = 0; i < RS; ++i) {
      const uint32_t wv[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint4 lo = xv[2 * e], hi = xv[2 * e + 1];
        a[i][0] = dp4a_us(wv[e] & 0x01010101u, lo.x, a[i][0]);
        a[i][1] = dp4a_us(wv[e] & 0x02020202u, lo.y, a[i][1]);
        a[i][2] = dp4a_us(wv[e] & 0x04040404u, lo.z, a[i][2]);
        a[i][3] = dp4a_us(wv[e] & 0x08080808u, lo.w, a[i][3]);
        a[i][4] = dp4a_us(wv[e] & 0x10101010u, hi.x, a[i][4]);
        a[i][5] = dp4a_us(wv[e] & 0x20202020u, hi.y, a[i][5]);
        a[i][6] = dp4a_us(wv[e] & 0x40404040u, hi.z, a[i][6]);
        a[i][7] = dp4a_us(wv[e] & 0x80808080u, hi.w, a[i][7]);
      }
    }
  };
  const uint8_t* wrow = wbase + static_cast<int64_t>(rb) * rowb + 16 * lj;
  const int8_t* xp = xs + 16 * lj;
  if (nr == RS) {
    for (int c = lj; c < nchunk; c += G) {
      uint4 w[RS];
#pragma unroll
      for (int i = 0; i < RS; ++i) w[i] = *reinterpret_cast<const uint4*>(wrow + i * rowb);
      body(w, xp);
      wrow += 16 * G;
      xp += 16 * G;
    }
  } else if (nr > 0) {
    for (int c = lj; c < nchunk; c += G) {
      uint4 w[RS];
#pragma unroll
      for (int i = 0; i < RS; ++i)
        w[i] = (i < nr) ? *reinterpret_cast<const uint4*>(wrow + i * rowb) : make_uint4(0u, 0u, 0u, 0u);
      body(w, xp);
      wrow += 16 * G;
      xp += 16 * G;
    }
  }
#pragma unroll
  for (int i = 0; i < RS; ++i) {
    int t = 0;
#pragma unroll
    for (int f = 0; f < 8; ++f) t += a[i][f] >> f;
#pragma unroll
    for (int o = G / 2; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    a[i][0] = t;
  }
#pragma unroll
  for (int i = 0; i < RS; ++i) {
    if (lj == i && i < nr) {
      const int64_t n = r + rb + i;
      const int accv = 2 * a[i][0] - xsum0;
      if (P.acc != nullptr) P.acc[n] = accv;
      if (P.y != nullptr) {
        float o = __fmul_rn(__int2float_rn(accv), gs0);
        if (P.resid != nullptr) o = __fadd_rn(load_y(P.resid, y_dtype, n), o);
        store_y(P.y, y_dtype, n, o);
      }
    }
  }
}

// Base-3 weights, M = 1: a warp owns R rows; lane l takes the 20-weight
// groups l, l + 32, ... of each.  Group g is one uint32 whose byte j holds
// the codes of weights 20g + 4i + j as base-3 digits i = 0..4.  The digits
// come out two bytes at a time in 16-bit lanes: floor(v / 3) = (v * 171) >> 9
// for every byte value v, and v - 3 floor(v / 3) is the digit, so digit i of
// the four bytes lines up four codes with the activation word at 20g + 4i
// for dp4a.  The code row is zero-padded past K (padding weights code 1).
// Rows [row0, row0 + R) of the chunk.
template <int R>
__device__ __forceinline__ void gs_task_t3(const uint8_t* wbase, int rc, int row0, int rowb, const int8_t* xs,
                                           int lane, int xsum0, float gs0, const GsProblem& P, int r, int y_dtype) {
  const int nr = min(R, rc - row0);
  const int nword = rowb / 4;
  const uint32_t* wb = reinterpret_cast<const uint32_t*>(wbase + static_cast<int64_t>(row0) * rowb);
  const uint32_t* x32 = reinterpret_cast<const uint32_t*>(xs);
  int a[R];
#pragma unroll
  for (int i = 0; i < R; ++i) a[i] = 0;
  for (int g = lane; g < nword; g += 32) {
    uint32_t xw[5];
#pragma unroll
    for (int d = 0; d < 5; ++d) xw[d] = x32[5 * g + d];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const uint32_t w = (i < nr) ? wb[i * nword + g] : 0u;
      uint32_t lo = w & 0x00FF00FFu, hi = (w >> 8) & 0x00FF00FFu;
#pragma unroll
      for (int d = 0; d < 5; ++d) {
        const uint32_t ql = ((lo * 171u) >> 9) & 0x007F007Fu, qh = ((hi * 171u) >> 9) & 0x007F007Fu;
        a[i] = dp4a_us((lo - 3u * ql) | ((hi - 3u * qh) << 8), xw[d], a[i]);
        lo = ql;
        hi = qh;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < R; ++i) a[i] = warp_sum(a[i]);
#pragma unroll
  for (int i = 0; i < R; ++i) {
    if (lane == i && i < nr) {
      const int64_t n = r + row0 + i;
      const int accv = a[i] - xsum0;
      if (P.acc != nullptr) P.acc[n] = accv;
      if (P.y != nullptr) {
        float o = __fmul_rn(__int2float_rn(accv), gs0);
        if (P.resid != nullptr) o = __fadd_rn(load_y(P.resid, y_dtype, n), o);
        store_y(P.y, y_dtype, n, o);
      }
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
        if (P.y != nullptr) {
          float o = __fmul_rn(__int2float_rn(accv), __fmul_rn(gamma, sc[m]));
          if (P.resid != nullptr) o = __fadd_rn(load_y(P.resid, y_dtype, idx), o);
          store_y(P.y, y_dtype, idx, o);
        }
      }
    }
}

// CW consumer warps + one activation warp.
// BITS (the weight format, 2 / 1 / 3 as GsParams::bits) is a template
// parameter so that each instantiation holds only its own contraction
// tasks: fewer code bytes in the consumers' loop, fewer instruction-cache
// misses.
template <int MT, int MAXP, int CW, int BITS>
__global__ void __launch_bounds__(CW * 32 + 32, 1) gemv_stream_kernel(const __grid_constant__ GsParams<MAXP> p) {
  static_assert(BITS == 2 || MT == 1, "1-bit and base-3 weights: one token");
  constexpr int kAll = CW * 32 + 32;
  extern __shared__ __align__(128) uint8_t smem[];
  static_assert(sizeof(GsHeader<MT, CW>) <= kGsHeader, "header too large");
  GsHeader<MT, CW>& H = *reinterpret_cast<GsHeader<MT, CW>*>(smem);
  const int xs_stride = MT * p.Kp_max;                       // one activation buffer
  int8_t* xsbuf = reinterpret_cast<int8_t*>(smem + kGsHeader);
  uint8_t* wslots = smem + kGsHeader + p.nxb * xs_stride;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int pb, rb, pe, re;
  gs_cta_start(p, blockIdx.x, pb, rb);
  gs_cta_start(p, blockIdx.x + 1, pe, re);
  if (blockIdx.x + 1 == gridDim.x) {
    pe = p.nprob;
    re = 0;
  }
  const int qlast = (re > 0) ? pe : pe - 1;
  auto seg_bounds = [&](int q, int& r0, int& r1) {
    r0 = (q == pb) ? rb : 0;
    r1 = (q == pe) ? re : p.prob[q].N;
  };
  auto shares_x = [&](int q) {   // segment q reuses segment q-1's quantised activations
    return q > pb && p.prob[q].x == p.prob[q - 1].x && p.prob[q].x2 == p.prob[q - 1].x2 &&
           p.prob[q].gain == p.prob[q - 1].gain && p.prob[q].K == p.prob[q - 1].K &&
           p.prob[q].x_scale == p.prob[q - 1].x_scale;
  };
  // Move a cursor `steps` chunks forward through the CTA's segments.
  auto advance = [&](GsCursor& c, int steps) {
    while (c.q <= qlast) {
      const int rc = p.prob[c.q].rc;
      if (c.r + steps * rc < c.r1) {   // stays in this segment (the usual case)
        c.r += steps * rc;
        return;
      }
      steps -= (c.r1 - c.r + rc - 1) / rc;
      ++c.q;
      if (c.q <= qlast) seg_bounds(c.q, c.r, c.r1);
    }
  };
  const int64_t esz = p.prequant ? 1 : (p.x_dtype == BITNET_BF16 ? 2 : 4);

  if (tid == 0) {
    for (int w = 0; w < CW; ++w)
      for (int s = 0; s < p.nslots; ++s) mbar_init(&H.wfull[w][s], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&H.xfull[b], 32);
      mbar_init(&H.xfree[b], CW);
    }
    mbar_init(&H.xcopy, 1);
    H.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &H.abort;

  GsCursor first{pb, 0, 0};
  if (pb <= qlast) seg_bounds(pb, first.r, first.r1);
  advance(first, 0);
  if (first.q > qlast) {   // empty share (more CTAs than rows)
    pdl_launch_dependents();
    return;
  }

  // ---- consumers: start this warp's weight stream before the dependency wait
  GsCursor cur = first, icur = first;
  int issued = 0;
  uint8_t* myslots = wslots + static_cast<size_t>(warp) * p.nslots * p.slot_bytes;
  auto issue = [&](int slot) {
    const GsProblem& Q = p.prob[icur.q];
    const int64_t rowb = gs_row_bytes(Q.K, BITS);
    const uint32_t bytes = static_cast<uint32_t>(min(Q.rc, icur.r1 - icur.r) * rowb);
    mbar_expect_tx(&H.wfull[warp][slot], bytes);
    bulk_g2s(myslots + slot * p.slot_bytes, Q.Wp + static_cast<int64_t>(icur.r) * rowb, bytes, &H.wfull[warp][slot]);
  };
  if (warp < CW) {
    advance(cur, warp);
    icur = cur;
    for (int i = 0; i < p.nslots && icur.q <= qlast; ++i) {
      if (lane == 0) issue(i);
      advance(icur, CW);
      ++issued;
    }
  }
  pdl_launch_dependents();
  pdl_wait();

  // Pre-quantised codes: copy one segment's codes into its buffer and form
  // their per-row sums (group of NT threads starting at thread tid0).
  int ncopy = 0;
  auto copy_codes = [&](const GsProblem& P, int8_t* xs, int Kp, float (&sc)[MT], int* qpart, int nt, int t0,
                        bool issuer) -> bool {
    if (issuer) {
      const uint32_t bytes = static_cast<uint32_t>(p.M * P.K);
      mbar_expect_tx(&H.xcopy, bytes);
      bulk_g2s(xs, P.x, bytes, &H.xcopy);
    }
    const bool got = gs_wait(&H.xcopy, ncopy & 1, p.limit_ns, abort_flag);
    if (!got && issuer) mbar_wait_bounded(&H.xcopy, ncopy & 1, p.limit_ns, nullptr);   // let it land
    ++ncopy;
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      int part = 0;
      if (got && m < p.M) {
        for (int k = (tid - t0) * 16; k < P.K; k += nt * 16) {
          const uint4 v = *reinterpret_cast<const uint4*>(xs + m * Kp + k);
          part = __dp4a(static_cast<int>(v.x), 0x01010101, part);
          part = __dp4a(static_cast<int>(v.y), 0x01010101, part);
          part = __dp4a(static_cast<int>(v.z), 0x01010101, part);
          part = __dp4a(static_cast<int>(v.w), 0x01010101, part);
        }
      }
      part = warp_sum(part);
      if (lane == 0) qpart[m * (nt / 32) + ((tid - t0) >> 5)] = part;
      sc[m] = (got && m < p.M) ? __ldg(P.x_scale + m) : 0.0f;
    }
    return got;
  };

  // ---- the first two activation versions, quantised by every warp (the
  // activation warp then has a whole segment to prepare each later one)
  bool ok = true;
  int q1 = pb + 1;                 // segment of version 1
  while (q1 <= qlast && shares_x(q1)) ++q1;
  const int ncoop = (q1 <= qlast && p.nxb == 2) ? 2 : 1;
  for (int cv = 0; cv < ncoop; ++cv) {
    const GsProblem& P = p.prob[cv == 0 ? pb : q1];
    int8_t* xs = xsbuf + cv * xs_stride;
    float sc[MT];
    const int Kp = gs_code_row(P.K, BITS);
    if (p.prequant) {
      ok = copy_codes(P, xs, Kp, sc, &H.q.qpart[0][0], kAll, 0, tid == CW * 32) && ok;
    } else {
      quant_rows<kAll, MT, 1, false, kGsBarAll, false>(static_cast<const char*>(P.x), p.x_dtype, P.K * esz, p.M,
                                                      P.K, P.gain, p.rms_eps, xs, Kp, H.q, sc, 0, p.blocked,
                                                      static_cast<const char*>(P.x2));
    }
    if constexpr (BITS == 3) {   // zero the code row's padding past K (no thread above wrote there)
      for (int k = P.K + tid; k < Kp; k += kAll) xs[k] = 0;
    }
    group_sync<kGsBarAll, kAll>();
    // the activation warp publishes the version; it reads the shared partials
    // before any warp can pass the next version's first barrier
    if (warp == CW) {
      if (lane == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          int t = 0;
          for (int w = 0; w < CW + 1; ++w) t += H.q.qpart[m][w];
          H.xsum[cv][m] = t;
          H.scale[cv][m] = sc[m];
        }
      }
      __syncwarp();
      mbar_arrive(&H.xfull[cv]);
    }
  }
  if (!ok && tid == 0 && !*abort_flag) {
    record_error(p.status, BITNET_ERR_TIMEOUT, 0x401u);
    *abort_flag = 1;
  }

  if (warp == CW) {
    // ============================================================ activations
    int v = ncoop - 1;
    for (int q = (ncoop == 2 ? q1 : pb) + 1; q <= qlast && ok && !*abort_flag; ++q) {
      if (shares_x(q)) continue;
      ++v;
      const int b = v % p.nxb;
      if (!gs_wait(&H.xfree[b], ((v / p.nxb) & 1) ^ 1u, p.limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      const GsProblem& P = p.prob[q];
      const int Kp = gs_code_row(P.K, BITS);
      int8_t* xs = xsbuf + b * xs_stride;
      float sc[MT];
      if (p.prequant) {
        if (!copy_codes(P, xs, Kp, sc, &H.qx.qpart[0][0], 32, CW * 32, lane == 0)) {
          ok = false;
          break;
        }
      } else {
        quant_rows<32, MT, 1, false, kGsBarX, false>(static_cast<const char*>(P.x), p.x_dtype, P.K * esz, p.M,
                                                     P.K, P.gain, p.rms_eps, xs, Kp, H.qx, sc, CW * 32,
                                                     p.blocked, static_cast<const char*>(P.x2));
      }
      if constexpr (BITS == 3)
        for (int k = P.K + lane; k < Kp; k += 32) xs[k] = 0;
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          H.xsum[b][m] = H.qx.qpart[m][0];
          H.scale[b][m] = sc[m];
        }
      }
      __syncwarp();
      mbar_arrive(&H.xfull[b]);
    }
    if (!ok && lane == 0 && !*abort_flag) {
      record_error(p.status, BITNET_ERR_TIMEOUT, 0x402u);
      *abort_flag = 1;
    }
    return;
  }

  // ================================================================== consumers
  float sc[MT];
  int xsum[MT];
  int v = -1, t = 0, slot = 0;
  uint32_t phase = 0;
  float gamma_next = 0.0f;
  for (int q = pb; q <= qlast && ok; ++q) {
    if (q == pb || !shares_x(q)) {
      if (v >= 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&H.xfree[v % p.nxb]);
      }
      ++v;
      if (!gs_wait(&H.xfull[v % p.nxb], (v / p.nxb) & 1, p.limit_ns, abort_flag)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        sc[m] = H.scale[v % p.nxb][m];
        xsum[m] = H.xsum[v % p.nxb][m];
      }
    }
    const GsProblem& P = p.prob[q];
    const int8_t* xs = xsbuf + (v % p.nxb) * xs_stride;
    const int Kp = gs_code_row(P.K, BITS);
    const float gamma = (q == pb) ? __ldg(P.gamma) : gamma_next;
    if (q < qlast) gamma_next = __ldg(p.prob[q + 1].gamma);   // in flight during this segment
    const float gs0 = __fmul_rn(gamma, sc[0]);
    const int nword = P.K / 16;      // 32-bit code words (16 weights) per row
    const int rowb = static_cast<int>(gs_row_bytes(P.K, BITS)), nchunk = rowb / 16;   // 16-byte chunks per row
    while (cur.q == q) {
      if (!gs_wait(&H.wfull[warp][slot], phase, p.limit_ns, abort_flag)) {
        ok = false;
        break;
      }
      const uint8_t* wb8 = myslots + slot * p.slot_bytes;
      const int rows = min(P.rc, cur.r1 - cur.r);
      const int r = cur.r;
      if constexpr (BITS == 3) {
        for (int row0 = 0; row0 < rows; row0 += 4)
          gs_task_t3<4>(wb8, rows, row0, rowb, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
      } else if constexpr (BITS == 1) {
        if (P.task == kGsTaskB1 + kGsTaskG8R2) {
          for (int row0 = 0; row0 < rows; row0 += 8)
            gs_task_lg_b1<8, 2>(wb8, rows, row0, rowb, nchunk, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
        } else if (P.task == kGsTaskB1 + kGsTaskG16R2) {
          for (int row0 = 0; row0 < rows; row0 += 4)
            gs_task_lg_b1<16, 2>(wb8, rows, row0, rowb, nchunk, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
        } else if (P.task == kGsTaskB1 + kGsTaskG16R1) {
          for (int row0 = 0; row0 < rows; row0 += 2)
            gs_task_lg_b1<16, 1>(wb8, rows, row0, rowb, nchunk, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
        } else {
          for (int row0 = 0; row0 < rows; ++row0)
            gs_task_lg_b1<32, 1>(wb8, rows, row0, rowb, nchunk, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
        }
      } else if (MT == 1 && P.task == kGsTaskG8R2) {
        for (int row0 = 0; row0 < rows; row0 += 8)
          gs_task_lg<8, 2>(wb8, rows, row0, rowb, nchunk, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
      } else if (MT == 1 && P.task == kGsTaskG16R2) {
        for (int row0 = 0; row0 < rows; row0 += 4)
          gs_task_lg<16, 2>(wb8, rows, row0, rowb, nchunk, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
      } else if (MT == 1 && P.task == kGsTaskG16R1) {
        for (int row0 = 0; row0 < rows; row0 += 2)
          gs_task_lg<16, 1>(wb8, rows, row0, rowb, nchunk, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
      } else if (MT == 1 && P.task == kGsTaskG32R1) {
        for (int row0 = 0; row0 < rows; ++row0)
          gs_task_lg<32, 1>(wb8, rows, row0, rowb, nchunk, xs, lane, xsum[0], gs0, P, r, p.y_dtype);
      } else {
        constexpr int R = (MT == 1) ? 4 : ((MT == 2) ? 2 : 1);
        const uint32_t* wbase = reinterpret_cast<const uint32_t*>(wb8);
        for (int row0 = 0; row0 < rows; row0 += R)
          gs_task_warp<R, MT>(wbase, rows, row0, nword, nword, xs, Kp, lane, xsum, sc, gamma, P, r, p.M,
                              p.y_dtype);
      }
      __syncwarp();
      if (icur.q <= qlast) {
        if (lane == 0) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          issue(slot);
        }
        advance(icur, CW);
        ++issued;
      }
      advance(cur, CW);
      ++t;
      if (++slot == p.nslots) {
        slot = 0;
        phase ^= 1u;
      }
    }
  }
  if (!ok) {
    if (lane == 0) {
      if (!*abort_flag) {
        record_error(p.status, BITNET_ERR_TIMEOUT, 0x403u);
        *abort_flag = 1;
      }
      // let this warp's weight copies still in flight land before the CTA exits
      for (int i = t; i < issued; ++i)
        mbar_wait_bounded(&H.wfull[warp][i % p.nslots], (i / p.nslots) & 1, p.limit_ns, nullptr);
    }
    __syncwarp();
  }
}

}  // namespace bitnet
