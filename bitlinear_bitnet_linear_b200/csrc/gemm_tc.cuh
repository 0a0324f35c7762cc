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

// Read the packed codes of one weight row for K block kb (32 bytes = 128
// weights) into 8 words; bytes past the row end (or rows past N) read as 0.
__device__ __forceinline__ void tc_load_row_block(const uint8_t* __restrict__ row, bool valid, int rowbytes,
                                                  int kb, int wvec, uint32_t (&w)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = 0u;
  if (!valid) return;
  const int off = kb * 32;
  const int avail = rowbytes - off;   // > 0, multiple of 4 (16 when wvec)
  if (wvec) {
    const uint4* p = reinterpret_cast<const uint4*>(row + off);
    const uint4 a = __ldg(p);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    if (avail >= 32) {
      const uint4 b = __ldg(p + 1);
      w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
  } else {
    const uint32_t* p = reinterpret_cast<const uint32_t*>(row + off);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (4 * i < avail) w[i] = __ldg(p + i);
  }
}

template <int BM, int SS, int AS>
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
    const int rowbytes = p.K / 4;
    const uint8_t* wrow = p.Wp + static_cast<int64_t>(valid ? n : 0) * rowbytes;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;

    uint32_t wb[kPD][8];
#pragma unroll
    for (int j = 0; j < kPD; ++j)
      if (j < KB) tc_load_row_block(wrow, valid, rowbytes, j, p.wvec, wb[j]);

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
              const uint32_t w = wb[j][g];
              codes[4 * g + 0] = w & 0x03030303u;
              codes[4 * g + 1] = (w >> 2) & 0x03030303u;
              codes[4 * g + 2] = (w >> 4) & 0x03030303u;
              codes[4 * g + 3] = (w >> 6) & 0x03030303u;
            }
            tmem_st_32x32b_x32(tmem + lane_base + kACol0 + 32u * a, codes);
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&afull[a]);
            if (kb + kPD < KB) tc_load_row_block(wrow, valid, rowbytes, kb + kPD, p.wvec, wb[j]);
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
            const int a = static_cast<int>(v[i]) - xsi;
            const int64_t idx = static_cast<int64_t>(m) * p.N + n;
            if (p.acc != nullptr) p.acc[idx] = a;
            if (p.y != nullptr) store_y(p.y, p.y_dtype, idx, __fmul_rn(__int2float_rn(a), gsi));
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
