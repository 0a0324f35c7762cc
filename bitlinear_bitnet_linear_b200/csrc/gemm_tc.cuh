// gemm_tc.cuh -- ternary x int8 GEMM on the 5th-generation tensor cores.
//
// acc[m,n] = sum_k x_q[m,k] * W_q[n,k];  y[m,n] = acc[m,n] * gamma * s_x[m]
//
// Swap-AB formulation: the MMA's A operand (M = 128 rows) is a tile of 128
// weight rows, its N dimension is a tile of BM tokens, so the accumulator
// D[n, m] lives in tensor memory with one weight row per TMEM lane.  The A
// operand is never staged in shared memory: converter warps read the packed
// 2-bit codes, expand them to one unsigned byte per weight (code c = q + 1 in
// {0, 1, 2}; two instructions per output word) and write them straight into
// tensor memory with tcgen05.st, where tcgen05.mma (kind::i8, A from TMEM,
// unsigned A x signed B) consumes them.  The offset is removed exactly in the
// epilogue: sum_k q x = sum_k c x - sum_k x  (the ternary dot product as
// "sum at +1 minus sum at -1", Hacker News thread on the b1.58 paper).
//
// Roles (192 threads):
//   warp 0       TMA producer: activation tiles [BM x 128 B], 128-byte swizzle
//   warp 1       TMEM allocator and single-thread MMA issuer
//   warps 2..5   converters (one weight row per thread), then the epilogue
// Pipeline: SS activation stages in shared memory and AS 32-column A buffers
// in TMEM, cycled independently.  mbarriers: full[s] (TMA bytes landed),
// sempty[s] (MMAs that read stage s completed; tcgen05.commit), afull[a] (128
// converter threads stored codes), aempty[a] (MMAs that read A buffer a
// completed), accf (all MMAs completed).  With BM <= 128 and AS = 4 a CTA
// holds 256 TMEM columns, so two CTAs share an SM and one's epilogue
// overlaps the other's main loop.
// Every wait is bounded; on expiry the kernel records BITNET_ERR_TIMEOUT,
// raises a CTA-wide abort flag, drains what it issued and frees TMEM.
#pragma once

#include "common.cuh"

namespace bitnet {

constexpr int kTcThreads = 192;
constexpr int kTcBK = 128;        // K elements (bytes) per stage = one 128-byte swizzle row
constexpr int kTcBN = 128;        // weight rows per CTA tile (MMA M)

struct TcParams {
  const uint8_t* Wp;
  const void* resid;     // [M, N] residual added to y (y_dtype), or nullptr
  const float* gamma;
  const float* x_scale;
  const int32_t* x_sum;
  void* y;
  int y_dtype;
  int32_t* acc;
  int M, K, N;
  int KB;        // ceil(K / 128)
  int wvec;      // 1: K % 64 == 0, weight rows 16-byte aligned
  uint64_t limit_ns;
  uint32_t* status;
};

__host__ __device__ constexpr uint32_t tc_tmem_cols(int BM, int AS) {
  const int need = BM + 32 * AS;
  return need <= 32 ? 32u : need <= 64 ? 64u : need <= 128 ? 128u : need <= 256 ? 256u : 512u;
}

template <int BM, int SS>
__host__ __device__ constexpr int tc_smem_bytes() {
  return 1024 /* alignment slack */ + SS * BM * kTcBK + 512 /* barriers, flags */;
}

// Read the packed codes of one weight row for K block kb (128 weights: 32
// bytes of 2-bit codes, or 16 bytes of 1-bit signs) into words w[0 .. 4 BITS);
// bytes past the row end (or rows past N) read as 0.
template <int BITS>
__device__ __forceinline__ void tc_load_row_block(const uint8_t* __restrict__ row, bool valid, int rowbytes,
                                                  int kb, int wvec, uint32_t (&w)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = 0u;
  if (!valid) return;
  const int off = kb * 16 * BITS;
  const int avail = rowbytes - off;   // > 0, multiple of 4 (16 when wvec)
  if (wvec) {
    const uint4* p = reinterpret_cast<const uint4*>(row + off);
    const uint4 a = __ldg(p);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    if (BITS == 2 && avail >= 32) {
      const uint4 b = __ldg(p + 1);
      w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
  } else {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(row + off);
#pragma unroll
    for (int i = 0; i < 4 * BITS; ++i)
      if (4 * i < avail) w[i] = __ldg(p + i);
  }
}

// The 16 unsigned bytes (one per weight, weights 16c .. 16c + 15 of the K
// block) of 16-byte chunk c, from the words of tc_load_row_block.  2-bit:
// field s of word c holds weights 16c + 4s .. + 3 (code c = q + 1).  1-bit:
// word c/2 holds weights 32(c/2) + 4s + j at bit 8j + s; chunk c takes
// s = 4(c % 2) .. + 3 (bit 1 for +1).
template <int BITS>
__device__ __forceinline__ uint4 tc_expand_chunk(const uint32_t (&w)[8], int c) {
  if constexpr (BITS == 2) {
    const uint32_t v = w[c];
    return make_uint4(v & 0x03030303u, (v >> 2) & 0x03030303u, (v >> 4) & 0x03030303u, (v >> 6) & 0x03030303u);
  } else {
    const uint32_t v = w[c >> 1] >> (4 * (c & 1));
    return make_uint4(v & 0x01010101u, (v >> 1) & 0x01010101u, (v >> 2) & 0x01010101u, (v >> 3) & 0x01010101u);
  }
}

// The exact dot product from the unsigned-code accumulator v and the code
// sum: 2-bit codes c = q + 1 give v - sum x; 1-bit signs b = (q + 1) / 2
// give 2 v - sum x.
template <int BITS>
__device__ __forceinline__ int tc_dot(uint32_t v, int xsum) {
  return BITS == 2 ? static_cast<int>(v) - xsum : 2 * static_cast<int>(v) - xsum;
}

template <int BM, int SS, int AS, int BITS = 2>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const TcParams p) {
  static_assert(BM % 16 == 0 && BM >= 16 && BM <= 256, "MMA N must be a multiple of 16 in [16, 256]");
  constexpr uint32_t kCols = tc_tmem_cols(BM, AS);
  constexpr uint32_t kACol0 = BM;                  // A buffer a at columns [BM + 32 a, BM + 32 a + 32)
  constexpr uint32_t kStageBytes = BM * kTcBK;
  constexpr uint32_t kIdesc = idesc_i8_us(kTcBN, BM);
  constexpr int kPD = 4;                           // converter prefetch depth (K blocks)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SS * kStageBytes);
  uint64_t* sempty = full + SS;
  uint64_t* afull = sempty + SS;
  uint64_t* aempty = afull + AS;
  uint64_t* accf = aempty + AS;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accf + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kTcBN;
  const int m0 = blockIdx.y * BM;
  const int KB = p.KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sempty[s], 1);
    }
    for (int a = 0; a < AS; ++a) {
      mbar_init(&afull[a], 128);
      mbar_init(&aempty[a], 1);
    }
    mbar_init(accf, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_x);
  if (warp == 1) {
    tmem_alloc(tmem_holder, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  auto fail = [&](uint32_t site) {
    record_error(p.status, BITNET_ERR_TIMEOUT, site);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      pdl_wait();   // activations come from the previous kernel
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % SS;
        const uint32_t ph = (kb / SS) & 1;
        if (!mbar_wait_bounded(&sempty[s], ph ^ 1u, p.limit_ns, abort_flag)) {
          if (!*abort_flag) fail(0x301u);
          break;
        }
        mbar_expect_tx(&full[s], kStageBytes);
        tma_load_2d(xs + s * kStageBytes, &tmap_x, kb * kTcBK, m0, &full[s]);
        ++issued;
      }
      if (*abort_flag) {
        // drain: let every copy already issued land before the CTA can exit
        for (int kb = max(0, issued - SS); kb < issued; ++kb)
          mbar_wait_bounded(&full[kb % SS], (kb / SS) & 1, p.limit_ns, nullptr);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int kb = 0; kb < KB && ok; ++kb) {
        const int s = kb % SS;
        const int a = kb % AS;
        if (!mbar_wait_bounded(&full[s], (kb / SS) & 1, p.limit_ns, abort_flag) ||
            !mbar_wait_bounded(&afull[a], (kb / AS) & 1, p.limit_ns, abort_flag)) {
          if (!*abort_flag) fail(0x302u);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t bdesc = smem_desc_k_sw128(smem_u32(xs + s * kStageBytes));
#pragma unroll
        for (int j = 0; j < kTcBK / 32; ++j) {
          // K step of 32 bytes: advance the descriptor start address by 32 B (>> 4 = 2)
          tc_mma_i8_ts(tmem, tmem + kACol0 + 32u * a + 8u * j, bdesc + 2ull * j, kIdesc,
                       (kb | j) != 0 ? 1u : 0u);
        }
        tc_commit(&sempty[s]);
        tc_commit(&aempty[a]);
      }
      // Completion of everything issued so far (also on abort: nothing may
      // still read TMEM when it is freed).
      tc_commit(accf);
      if (!ok) mbar_wait_bounded(accf, 0, p.limit_ns, nullptr);
    }
  } else {
    // ------------------------------------------------------------ converters
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;
    const int n = n0 + row;
    const bool valid = n < p.N;
    const int rowbytes = p.K * BITS / 8;
    const uint8_t* wrow = p.Wp + static_cast<int64_t>(valid ? n : 0) * rowbytes;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;

    uint32_t wb[kPD][8];
#pragma unroll
    for (int j = 0; j < kPD; ++j)
      if (j < KB) tc_load_row_block<BITS>(wrow, valid, rowbytes, j, p.wvec, wb[j]);

    bool ok = true;
    for (int kb0 = 0; kb0 < KB && ok; kb0 += kPD) {
#pragma unroll
      for (int j = 0; j < kPD; ++j) {
        const int kb = kb0 + j;
        if (kb < KB && ok) {
          const int a = kb % AS;
          const uint32_t ph = (kb / AS) & 1;
          if (!mbar_wait_bounded(&aempty[a], ph ^ 1u, p.limit_ns, abort_flag)) {
            if (!*abort_flag) fail(0x303u);
            ok = false;
          }
          // all lanes of the warp take the same branch below: waits return
          // together unless aborting, and tcgen05.st is warp-collective
          if (__all_sync(0xffffffffu, ok)) {
            uint32_t codes[32];
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              const uint4 c4 = tc_expand_chunk<BITS>(wb[j], g);
              codes[4 * g + 0] = c4.x;
              codes[4 * g + 1] = c4.y;
              codes[4 * g + 2] = c4.z;
              codes[4 * g + 3] = c4.w;
            }
            tmem_st_32x32b_x32(tmem + lane_base + kACol0 + 32u * a, codes);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&afull[a]);
            if (kb + kPD < KB) tc_load_row_block<BITS>(wrow, valid, rowbytes, kb + kPD, p.wvec, wb[j]);
          } else {
            ok = false;
          }
        }
      }
    }

    // ------------------------------------------------------------ epilogue
    if (ok && mbar_wait_bounded(accf, 0, p.limit_ns, abort_flag)) {
      tc_fence_after();
      pdl_wait();   // token scales and sums come from the previous kernel
      pdl_launch_dependents();
      const float gamma = __ldg(p.gamma);
      const float* __restrict__ xsc = p.x_scale;
      const int32_t* __restrict__ xsm = p.x_sum;
#pragma unroll 1
      for (int c0 = 0; c0 < BM; c0 += 32) {
        if (m0 + c0 >= p.M) break;   // warp-uniform
        // lane i fetches token (m0 + c0 + i)'s constants once; shuffled below
        const int mi = m0 + c0 + lane;
        float gs = 0.0f;
        int xsum = 0;
        if (mi < p.M) {
          gs = __fmul_rn(gamma, __ldg(xsc + mi));
          xsum = __ldg(xsm + mi);
        }
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + lane_base + static_cast<uint32_t>(c0), v);
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float gsi = __shfl_sync(0xffffffffu, gs, i);
          const int xsi = __shfl_sync(0xffffffffu, xsum, i);
          const int m = m0 + c0 + i;
          if (valid && m < p.M) {
            const int a = tc_dot<BITS>(v[i], xsi);
            const int64_t idx = static_cast<int64_t>(m) * p.N + n;
            if (p.acc != nullptr) p.acc[idx] = a;
            if (p.y != nullptr) {
              float o = __fmul_rn(__int2float_rn(a), gsi);
              if (p.resid != nullptr) o = __fadd_rn(load_y(p.resid, p.y_dtype, idx), o);
              store_y(p.y, p.y_dtype, idx, o);
            }
          }
        }
      }
    } else if (ok) {
      if (!*abort_flag) fail(0x304u);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// ---------------------------------------------------------------------------
// Persistent variant (M > 64): one CTA per SM walks output tiles of 256
// weight rows x BM = 128 tokens.  Each 128-wide K block feeds two M = 128
// MMAs (the two weight-row halves) that share one activation stage, halving
// the L2 traffic per MAC of a 128-row tile.
// A operand: the converters expand the 2-bit codes to one unsigned byte per
// weight and write them to TMEM with tcgen05.st; the MMAs read A from there
// (the TS form), so shared memory carries only the TMA-loaded activation
// tiles (B).  With both operands in shared memory, one 128x128x32 int8 MMA
// alone reads 8 KB in its 64-cycle slot, the SM's whole shared-memory
// bandwidth, before any converter store or TMA write.
// TMEM (512 columns): three accumulator slots of BM columns, then AS A
// stages of 64 columns (weight-row half h at +32 h, 8 columns per 32-byte K
// step).  Tile i accumulates its halves in slots 2i mod 3 and (2i + 1) mod
// 3; tile i + 1 takes the third slot and tile i's first, so its MMAs start
// as soon as the epilogue has read tile i's first half, while the epilogue
// goes on with the second.
// Roles (576 threads):
//   warp 0        TMA producer, running ahead across tiles (SS stages)
//   warp 1        TMEM allocator and single-thread MMA issuer
//   warps 2..9    converters: one weight row per thread, rows of TMEM lane
//                 quadrant w % 4 in half (w - 2) / 4 (a warp reaches only
//                 lanes [32 (w % 4), 32 (w % 4) + 32))
//   warps 10..17  epilogue: tokens [64 t, 64 t + 64), t = (w - 10) / 4, of
//                 both halves, lane quadrant w % 4
// Pipeline waits suspend in hardware (try_wait with a time hint), so warps
// with nothing to do take no issue slots from the others; only the MMA
// issuer, on the critical path, spins on its operand barriers.
// Barriers: full/sempty (activation stages), afull/aempty (A stages; 256
// converter arrivals), dfull (all MMAs of a tile done), dfree[s] (8 epilogue
// warps done reading slot s), mdone (every MMA issued has completed, before
// TMEM is freed).
// ---------------------------------------------------------------------------
constexpr int kTpRows = 256;
constexpr int kTpThreads = 18 * 32;

template <int BM, int SS>
__host__ __device__ constexpr int tp_smem_bytes() {
  return 1024 /* alignment slack */ + SS * BM * kTcBK + 1024 /* barriers, flags */;
}

template <int BM, int SS, int AS, int BITS = 2>
__global__ void __launch_bounds__(kTpThreads, 1)
    tc_gemm_persistent_kernel(const __grid_constant__ CUtensorMap tmap_x, const TcParams p) {
  static_assert(BM == 128 && 3 * BM + 64 * AS <= 512, "the accumulator slots and A stages fit 512 TMEM columns");
  constexpr uint32_t kCols = 512;
  constexpr uint32_t kACol0 = 3 * BM;                  // A stage a at [3 BM + 64 a, 3 BM + 64 a + 64)
  constexpr uint32_t kStageBytes = BM * kTcBK;
  constexpr uint32_t kIdesc = idesc_i8_us(kTcBN, BM);
  constexpr int kPD = 4;                               // converter prefetch depth (K blocks)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* xs = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SS * kStageBytes);
  uint64_t* sempty = full + SS;
  uint64_t* afull = sempty + SS;
  uint64_t* aempty = afull + AS;
  uint64_t* dfull = aempty + AS;
  uint64_t* dfree = dfull + 1;
  uint64_t* mdone = dfree + 3;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = p.KB;
  const int n_tiles = (p.N + kTpRows - 1) / kTpRows;
  const int tiles = n_tiles * ((p.M + BM - 1) / BM);
  const int G = gridDim.x;
  // local tile i of this CTA: global tile blockIdx.x + i * G; tiles of one
  // token block are adjacent, so CTAs running together share activation tiles
  const int my_tiles = blockIdx.x < tiles ? (tiles - 1 - blockIdx.x) / G + 1 : 0;
  auto tile_m0 = [&](int i) { return ((blockIdx.x + i * G) / n_tiles) * BM; };
  auto tile_n0 = [&](int i) { return ((blockIdx.x + i * G) % n_tiles) * kTpRows; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < SS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sempty[s], 1);
    }
    for (int a = 0; a < AS; ++a) {
      mbar_init(&afull[a], 256);
      mbar_init(&aempty[a], 1);
    }
    mbar_init(dfull, 1);
    for (int s = 0; s < 3; ++s) mbar_init(&dfree[s], 8);
    mbar_init(mdone, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_x);
  if (warp == 1) {
    tmem_alloc(tmem_holder, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  auto fail = [&](uint32_t site) {
    record_error(p.status, BITNET_ERR_TIMEOUT, site);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      pdl_wait();   // activations come from the previous kernel
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int m0 = tile_m0(i);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % SS;
          if (!mbar_wait_sleep(&sempty[s], ((g / SS) & 1) ^ 1u, p.limit_ns, abort_flag)) {
            if (!*abort_flag) fail(0x311u);
            ok = false;
            break;
          }
          mbar_expect_tx(&full[s], kStageBytes);
          tma_load_2d(xs + s * kStageBytes, &tmap_x, kb * kTcBK, m0, &full[s]);
        }
      }
      if (!ok) {
        // let every copy already issued land before the CTA can exit
        for (int j = max(0, g - SS); j < g; ++j) mbar_wait_bounded(&full[j % SS], (j / SS) & 1, p.limit_ns, nullptr);
      }
    }
    pdl_launch_dependents();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int g = 0;
      uint32_t slot_par = 0;   // bit s = parity of the uses of slot s so far
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int s0 = (2 * i) % 3, s1 = (2 * i + 1) % 3;
        // the epilogue has read what earlier tiles left in both slots
        if (!mbar_wait_sleep(&dfree[s0], ((slot_par >> s0) & 1u) ^ 1u, p.limit_ns, abort_flag) ||
            !mbar_wait_sleep(&dfree[s1], ((slot_par >> s1) & 1u) ^ 1u, p.limit_ns, abort_flag)) {
          if (!*abort_flag) fail(0x312u);
          ok = false;
          break;
        }
        slot_par ^= (1u << s0) | (1u << s1);
        tc_fence_after();
        const uint32_t d0 = tmem + static_cast<uint32_t>(s0 * BM);   // weight-row half 0
        const uint32_t d1 = tmem + static_cast<uint32_t>(s1 * BM);   // weight-row half 1
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % SS;
          const int a = g % AS;
          // the issuer is the critical path: it spins (one thread), the others sleep
          if (!mbar_wait_bounded(&full[s], (g / SS) & 1, p.limit_ns, abort_flag) ||
              !mbar_wait_bounded(&afull[a], (g / AS) & 1, p.limit_ns, abort_flag)) {
            if (!*abort_flag) fail(0x313u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = smem_desc_k_sw128(smem_u32(xs + s * kStageBytes));
          const uint32_t a0 = tmem + kACol0 + 64u * static_cast<uint32_t>(a);
#pragma unroll
          for (int j = 0; j < kTcBK / 32; ++j) {
            // K step of 32 bytes: 8 TMEM columns of A, 32 B of the B descriptor (>> 4 = 2)
            const uint32_t acc = (kb | j) != 0 ? 1u : 0u;
            tc_mma_i8_ts(d0, a0 + 8u * j, bdesc + 2ull * j, kIdesc, acc);
            tc_mma_i8_ts(d1, a0 + 32u + 8u * j, bdesc + 2ull * j, kIdesc, acc);
          }
          tc_commit(&sempty[s]);
          tc_commit(&aempty[a]);
        }
        if (ok) tc_commit(dfull);
      }
      // every MMA issued has completed before TMEM can be freed
      tc_commit(mdone);
      mbar_wait_bounded(mdone, 0, p.limit_ns, nullptr);
    }
    pdl_launch_dependents();
  } else if (warp < 10) {
    // ------------------------------------------------------------ converters
    const int h = (warp - 2) >> 2;                     // weight-row half
    const int row = h * 128 + (warp & 3) * 32 + lane;  // A row of the 256-row tile
    const uint32_t a_lane_col = (static_cast<uint32_t>((warp & 3) * 32) << 16) + kACol0 + 32u * h;
    const int rowbytes = p.K * BITS / 8;
    const int total = my_tiles * KB;
    uint32_t wb[kPD][8];
    auto load = [&](int gi, uint32_t (&w)[8]) {
      const int i = gi / KB, kb = gi - i * KB;
      const int n = tile_n0(i) + row;
      const bool valid = n < p.N;
      tc_load_row_block<BITS>(p.Wp + static_cast<int64_t>(valid ? n : 0) * rowbytes, valid, rowbytes, kb, p.wvec,
                              w);
    };
#pragma unroll
    for (int j = 0; j < kPD; ++j)
      if (j < total) load(j, wb[j]);
    bool ok = true;
    for (int g0 = 0; g0 < total && ok; g0 += kPD) {
#pragma unroll
      for (int j = 0; j < kPD; ++j) {
        const int g = g0 + j;
        if (g < total && ok) {
          const int a = g % AS;
          if (!mbar_wait_sleep(&aempty[a], ((g / AS) & 1) ^ 1u, p.limit_ns, abort_flag)) {
            if (!*abort_flag) fail(0x314u);
            ok = false;
          }
          // tcgen05.st is warp-collective: the warp goes on only together
          // (the waits return together unless aborting)
          if (__all_sync(0xffffffffu, ok)) {
            uint32_t codes[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {   // chunk c: weights 16c .. 16c + 15 of the K block
              const uint4 c4 = tc_expand_chunk<BITS>(wb[j], c);
              codes[4 * c + 0] = c4.x;
              codes[4 * c + 1] = c4.y;
              codes[4 * c + 2] = c4.z;
              codes[4 * c + 3] = c4.w;
            }
            tmem_st_32x32b_x32(tmem + a_lane_col + 64u * static_cast<uint32_t>(a), codes);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&afull[a]);
            if (g + kPD < total) load(g + kPD, wb[j]);
          } else {
            ok = false;
          }
        }
      }
    }
    pdl_launch_dependents();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                     // TMEM lane quadrant
    const int tok0 = ((warp - 10) >> 2) * 64;   // first token of this warp in the tile
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    constexpr int kChunks = 2;                  // 64 tokens in chunks of 32
    const bool fast = p.y != nullptr && p.acc == nullptr && p.resid == nullptr && p.y_dtype == BITNET_BF16 &&
                      p.K <= 32768;
    pdl_wait();   // token scales and sums come from the previous kernel
    const float gamma = __ldg(p.gamma);
    const float* __restrict__ xsc = p.x_scale;
    const int32_t* __restrict__ xsm = p.x_sum;
    for (int i = 0; i < my_tiles; ++i) {
      const int m0 = tile_m0(i) + tok0;   // this warp's first token
      // chunks of 32 tokens holding tokens below M (warp-uniform)
      const int nc = min(kChunks, (max(0, p.M - m0) + 31) / 32);
      // lane l holds token (m0 + 32 c + l)'s scale and code sum: loaded before
      // the accumulators are ready, shuffled out below
      float gs[kChunks];
      int xsum[kChunks];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        const int mi = m0 + 32 * c + lane;
        gs[c] = 0.0f;
        xsum[c] = 0;
        if (mi < p.M) {
          gs[c] = __fmul_rn(gamma, __ldg(xsc + mi));
          xsum[c] = __ldg(xsm + mi);
        }
      }
      const bool got = mbar_wait_sleep(dfull, i & 1, p.limit_ns, abort_flag);
      if (!got && !*abort_flag) fail(0x315u);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      if (i + 1 == my_tiles) pdl_launch_dependents();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {                    // weight-row half, its slot
        const int slot = (2 * i + h) % 3;
        const int n = tile_n0(i) + h * 128 + q * 32 + lane;
        const bool valid = n < p.N;
        const uint32_t dcol = static_cast<uint32_t>(slot * BM + tok0);
        if (nc == 0) {
          // no token of this warp in the tile: hand the slot back at once
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dfree[slot]);
        }
        // A rolled loop over the 32-token chunks keeps the (unrolled) chunk
        // body in the instruction cache: fully unrolled, the epilogue is
        // straight-line code that runs once per tile and misses on every fetch.
#pragma unroll 1
        for (int c = 0; c < nc; ++c) {
          const float gsc = c == 0 ? gs[0] : gs[1];
          const int xsc_ = c == 0 ? xsum[0] : xsum[1];
          uint32_t v[32];
          tmem_ld_32x32b_x32(tmem + lane_base + dcol + static_cast<uint32_t>(32 * c), v);
          tc_wait_ld();
          if (c + 1 == nc) {
            // the last read of this slot has landed: the MMAs of the next
            // tile may start while this warp stores
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&dfree[slot]);
          }
          if (fast) {
            // |acc| <= 128 K <= 2^22: conversions on the integer pipes (the
            // conversion unit would otherwise bound the epilogue)
            uint16_t* yb = static_cast<uint16_t*>(p.y) + static_cast<int64_t>(m0 + 32 * c) * p.N + n;
#pragma unroll
            for (int t = 0; t < 32; ++t) {
              const float gst = __shfl_sync(0xffffffffu, gsc, t);
              const int xst = __shfl_sync(0xffffffffu, xsc_, t);
              if (valid && m0 + 32 * c + t < p.M)
                yb[static_cast<int64_t>(t) * p.N] =
                    bf16_bits_rne(__fmul_rn(small_int_to_float(tc_dot<BITS>(v[t], xst)), gst));
            }
          } else {
#pragma unroll
            for (int t = 0; t < 32; ++t) {
              const float gst = __shfl_sync(0xffffffffu, gsc, t);
              const int xst = __shfl_sync(0xffffffffu, xsc_, t);
              const int m = m0 + 32 * c + t;
              if (valid && m < p.M) {
                const int acc = tc_dot<BITS>(v[t], xst);
                const int64_t idx = static_cast<int64_t>(m) * p.N + n;
                if (p.acc != nullptr) p.acc[idx] = acc;
                if (p.y != nullptr) {
                  float o = __fmul_rn(__int2float_rn(acc), gst);
                  if (p.resid != nullptr) o = __fadd_rn(load_y(p.resid, p.y_dtype, idx), o);
                  store_y(p.y, p.y_dtype, idx, o);
                }
              }
            }
          }
        }
      }
    }
    pdl_launch_dependents();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// Watchdog self-test: wait on a barrier that nothing completes.
__global__ void watchdog_selftest_kernel(uint64_t limit_ns, uint32_t* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait_bounded(&bar, 0, limit_ns, nullptr)) record_error(status, BITNET_ERR_TIMEOUT, 0x3ffu);
  }
}

}  // namespace bitnet
