// bitnet.cu -- the C ABI of libbitnet.so (declared in include/bitnet.h):
// argument validation, path selection and kernel launches.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <new>
#include <vector>
#include <mutex>

#include "act.cuh"
#include "common.cuh"
#include "gemm_tc.cuh"
#include "gemv.cuh"
#include "gemv_stream.cuh"
#include "weights.cuh"

using namespace bitnet;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kGemvMaxM = 4;
constexpr size_t kWsHeader = sizeof(WsHeader);

std::atomic<uint64_t> g_limit_ns{2000000000ull};

struct DeviceInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
  int max_smem_optin = 0;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bitnet_status cuda_status(cudaError_t e) { return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA; }

bitnet_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return BITNET_ERR_UNSUPPORTED;
  }
  if (dev < 0 || dev >= kMaxDevices) return BITNET_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    d.init = true;
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaGetLastError();
    d.ok = (major == 10 && minor == 0 && d.sms > 0);
  }
  if (!d.ok) return BITNET_ERR_UNSUPPORTED;
  *out = &d;
  return BITNET_OK;
}

bitnet_status get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode != nullptr) return BITNET_OK;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr) {
    cudaGetLastError();
    return BITNET_ERR_CUDA;
  }
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return BITNET_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bitnet_status check_shape(int64_t M, int64_t K, int64_t N) {
  if (M < 1 || N < 1 || K < 16 || (K % 16) != 0) return BITNET_ERR_SHAPE;
  const int64_t lim = (int64_t(1) << 31) - 1;
  if (M > lim || N > lim || K > lim) return BITNET_ERR_SHAPE;
  if (N * K >= (int64_t(1) << 39) || M * K >= (int64_t(1) << 39) || M * N >= (int64_t(1) << 39))
    return BITNET_ERR_SHAPE;
  return BITNET_OK;
}

// Launch with programmatic stream serialisation allowed.
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device):
// the attribute call is host work that must not recur on every launch (and
// must not be needed inside a stream capture once warmed up).
template <typename Kern>
cudaError_t allow_smem(Kern kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  struct Entry {
    const void* fn;
    int dev;
    size_t bytes;
  };
  static Entry cache[256];
  static int used = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const void* fn = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lk(g_mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].fn == fn && cache[i].dev == dev) {
      if (cache[i].bytes >= bytes) return cudaSuccess;
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(bytes));
      if (e == cudaSuccess) cache[i].bytes = bytes;
      return e;
    }
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess && used < 256) cache[used++] = Entry{fn, dev, bytes};
  return e;
}

int elementwise_grid(int64_t work, const DeviceInfo* d) {
  const int64_t g = (work + 255) / 256;
  const int64_t cap = static_cast<int64_t>(d->sms) * 16;
  return static_cast<int>(g < 1 ? 1 : (g > cap ? cap : g));
}

// Workspace carve-up for the linear calls.
struct LinearWs {
  uint32_t* status;
  int8_t* xq;
  float* scale;
  int32_t* sum;
};
size_t linear_ws_bytes(int64_t M, int64_t K) {
  return kWsHeader + round_up(static_cast<size_t>(M * K), 256) + 2 * round_up(static_cast<size_t>(M) * 4, 256);
}
LinearWs carve(void* ws, int64_t M, int64_t K) {
  LinearWs w;
  uint8_t* b = static_cast<uint8_t*>(ws);
  w.status = reinterpret_cast<uint32_t*>(b);
  b += kWsHeader;
  w.xq = reinterpret_cast<int8_t*>(b);
  b += round_up(static_cast<size_t>(M * K), 256);
  w.scale = reinterpret_cast<float*>(b);
  b += round_up(static_cast<size_t>(M) * 4, 256);
  w.sum = reinterpret_cast<int32_t*>(b);
  return w;
}

// ---------------------------------------------------------------------------
// GEMV launch planning.
// ---------------------------------------------------------------------------
struct GemvPlan {
  int MT, R, grid, smem;
  GemvParams p;
};

bitnet_status plan_gemv(const DeviceInfo* d, int64_t M, int64_t K, int64_t N, GemvPlan& pl) {
  if (M > kGemvMaxM) return BITNET_ERR_UNSUPPORTED;
  GemvParams& p = pl.p;
  pl.MT = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.N = static_cast<int>(N);
  p.Kp = static_cast<int>(round_up(static_cast<size_t>(K), 64));
  p.bulk = (K % 64 == 0) ? 1 : 0;
  p.wrow = p.bulk ? static_cast<int>(K / 4) : p.Kp / 4;
  // Two CTAs per SM: each is latency-bound on its own, two overlap.
  const int64_t cap = 2 * static_cast<int64_t>(d->sms);
  const int grid = static_cast<int>(N < cap ? N : cap);
  pl.grid = grid;
  p.rows_base = static_cast<int>(N / grid);
  p.rows_extra = static_cast<int>(N % grid);
  const int rows_cta = p.rows_base + (p.rows_extra ? 1 : 0);
  // rows per warp task: enough tasks for all eight warps, more ILP when rows abound
  if (rows_cta <= kGvWarps) pl.R = 1;
  else if (rows_cta <= 2 * kGvWarps) pl.R = 2;
  else pl.R = K <= 4096 ? 4 : (K <= 8192 ? 2 : 1);
  if (pl.MT == 4 && pl.R == 4) pl.R = 2;
  const int xbytes = pl.MT * p.Kp;
  // Prefer a footprint that lets the next call's CTAs co-reside (PDL
  // overlap); grow only when two stages would not fit.
  const int budget_soft = 96 * 1024;
  const int budget_hard = d->max_smem_optin;
  int stage_rows = kGvWarps * pl.R;
  if (stage_rows > rows_cta) stage_rows = rows_cta;
  const int stage_bytes = stage_rows * p.wrow;
  const int nst = (rows_cta + stage_rows - 1) / stage_rows;
  int room = budget_soft - kGvHeader - xbytes;
  if (room < 2 * stage_bytes && nst > 1) room = budget_hard - kGvHeader - xbytes;
  int stages = room / stage_bytes;
  if (stages > kGvMaxStages) stages = kGvMaxStages;
  if (stages > nst) stages = nst;
  if (stages < 1) return BITNET_ERR_UNSUPPORTED;
  p.stage_rows = stage_rows;
  p.stages = stages;
  pl.smem = kGvHeader + xbytes + stages * stage_bytes;
  if (pl.smem > budget_hard) return BITNET_ERR_UNSUPPORTED;
  return BITNET_OK;
}

template <int MT, int R, bool FUSED>
cudaError_t run_gemv_t(const GemvPlan& pl, cudaStream_t st) {
  auto k = gemv_kernel<MT, R, FUSED>;
  cudaError_t e = allow_smem(k, pl.smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(pl.grid), dim3(kGvThreads), pl.smem, st, pl.p);
}

template <bool FUSED>
cudaError_t run_gemv(const GemvPlan& pl, cudaStream_t st) {
  switch (pl.MT * 10 + pl.R) {
    case 14: return run_gemv_t<1, 4, FUSED>(pl, st);
    case 12: return run_gemv_t<1, 2, FUSED>(pl, st);
    case 11: return run_gemv_t<1, 1, FUSED>(pl, st);
    case 22: return run_gemv_t<2, 2, FUSED>(pl, st);
    case 24: return run_gemv_t<2, 4, FUSED>(pl, st);
    case 21: return run_gemv_t<2, 1, FUSED>(pl, st);
    case 42: return run_gemv_t<4, 2, FUSED>(pl, st);
    case 41: return run_gemv_t<4, 1, FUSED>(pl, st);
    default: return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------------------
// Streaming GEMV (one or many problems, K % 64 == 0).
// ---------------------------------------------------------------------------
struct StreamProblem {
  const void* x;
  const uint8_t* Wp;
  const float* gamma;
  const float* gain;
  const float* x_scale;
  void* y;
  int32_t* acc;
  int64_t K, N;
  const void* x2;      // up projection of a ReLU^2-gated input (x is the gate), or nullptr
  const void* resid;   // residual added to y, or nullptr
};

template <int MAXP>
struct StreamPlan {
  int MT, grid, smem;
  GsParams<MAXP> p;
};

template <int MAXP>
bitnet_status plan_stream(const DeviceInfo* d, const StreamProblem* pr, int count, int64_t M, int x_dtype,
                          bool prequant, float rms_eps, int y_dtype, StreamPlan<MAXP>& pl, int bits = 2) {
  if (count < 1 || count > MAXP || M < 1 || M > kGemvMaxM) return BITNET_ERR_UNSUPPORTED;
  GsParams<MAXP>& p = pl.p;
  pl.MT = M <= 1 ? 1 : (M <= 2 ? 2 : 4);
  p.nprob = count;
  p.M = static_cast<int>(M);
  p.x_dtype = x_dtype;
  p.y_dtype = y_dtype;
  p.prequant = prequant ? 1 : 0;
  p.rms_eps = rms_eps;
  int64_t total = 0, max_rowb = 0, Kmax = 0, xmax = 0;
  const int64_t esz = prequant ? 1 : (x_dtype == BITNET_BF16 ? 2 : 4);
  p.bits = bits;
  for (int i = 0; i < count; ++i) {
    // 16-byte packed rows: K % 64 (2-bit), K % 128 (1-bit); base-3 rows are padded
    if ((bits == 2 && pr[i].K % 64 != 0) || (bits == 1 && pr[i].K % 128 != 0)) return BITNET_ERR_UNSUPPORTED;
    total += pr[i].N * gs_row_bytes(pr[i].K, bits);
    max_rowb = std::max<int64_t>(max_rowb, gs_row_bytes(pr[i].K, bits));
    Kmax = std::max<int64_t>(Kmax, gs_code_row(static_cast<int>(pr[i].K), bits));
    xmax = std::max<int64_t>(xmax, M * pr[i].K * esz);
  }
  p.total_bytes = total;
  // One CTA per SM.  A long stream (many calls in one launch) takes the whole
  // shared memory for the consumers' rings; a short one (a single decode
  // call) keeps a footprint that lets the next call's CTAs start beside it.
  const bool big = total >= (int64_t(32) << 20);
  int64_t grid = big ? d->sms : std::min<int64_t>(d->sms, (total + 4095) / 4096);
  if (grid < 1) grid = 1;
  pl.grid = static_cast<int>(grid);
  const int64_t per_cta = (total + grid - 1) / grid;
  p.Kp_max = static_cast<int>(Kmax);
  // single-token activations are stored block-permuted for the lane-group
  // tasks; pre-quantised codes are copied as they are (warp tasks)
  p.blocked = (pl.MT == 1 && !prequant && bits != 3) ? (bits == 2 ? 1 : 2) : 0;
  // 1-bit and base-3 GEMV: one token, raw activations
  if (bits != 2 && (pl.MT != 1 || prequant)) return BITNET_ERR_UNSUPPORTED;
  (void)xmax;
  // Shapes, most preferred first: (activation buffers, slots per warp, budget).
  // Two activation buffers let the activation warp run a segment ahead.
  struct Shape {
    int nxb, nslots;
    int64_t budget;
  };
  const int64_t small_budget = big ? d->max_smem_optin : 64 * 1024;
  const Shape shapes[] = {{2, 2, small_budget},
                          {2, 2, d->max_smem_optin},
                          {1, 2, d->max_smem_optin},
                          {2, 1, d->max_smem_optin},
                          {1, 1, d->max_smem_optin}};
  int64_t fixed = 0, slot = 0;
  int nslots = 0;
  for (const Shape& sh : shapes) {
    fixed = kGsHeader + sh.nxb * pl.MT * Kmax;
    slot = (sh.budget - fixed) / (kGsCW * sh.nslots) / 128 * 128;
    if (slot >= max_rowb) {
      p.nxb = sh.nxb;
      nslots = sh.nslots;
      break;
    }
  }
  if (nslots == 0) return BITNET_ERR_UNSUPPORTED;
  p.slot_bytes = static_cast<int>(slot);
  p.nslots = nslots;
  int64_t byte0 = 0;
  for (int i = 0; i < count; ++i) {
    GsProblem& g = p.prob[i];
    g.x = pr[i].x;
    g.Wp = pr[i].Wp;
    g.gamma = pr[i].gamma;
    g.gain = pr[i].gain;
    g.x_scale = pr[i].x_scale;
    g.y = pr[i].y;
    g.acc = pr[i].acc;
    g.x2 = pr[i].x2;
    g.resid = pr[i].resid;
    g.K = static_cast<int>(pr[i].K);
    g.N = static_cast<int>(pr[i].N);
    const int64_t rowb = gs_row_bytes(pr[i].K, bits);
    int64_t rc = slot / rowb;
    // a short stream: about one chunk per consumer warp
    if (!big) rc = std::min<int64_t>(rc, ((per_cta + rowb - 1) / rowb + kGsCW - 1) / kGsCW);
    rc = std::max<int64_t>(1, std::min<int64_t>(rc, pr[i].N));
    int task;
    if (bits == 3) {
      task = kGsTaskT3;
      if (rc >= 4) rc -= rc % 4;
    } else if (p.blocked) {
      // the largest lane-group task whose rows fit the chunk
      task = rc >= 8 ? kGsTaskG8R2 : (rc >= 4 ? kGsTaskG16R2 : (rc >= 2 ? kGsTaskG16R1 : kGsTaskG32R1));
      const int64_t unit = task == kGsTaskG8R2 ? 8 : (task == kGsTaskG16R2 ? 4 : (task == kGsTaskG16R1 ? 2 : 1));
      rc -= rc % unit;
      if (bits == 1) task += kGsTaskB1;
    } else {
      task = kGsTaskWarp;
      const int64_t unit = pl.MT == 1 ? 4 : (pl.MT == 2 ? 2 : 1);
      if (rc >= unit) rc -= rc % unit;
    }
    g.rc = static_cast<int>(rc);
    g.task = task;
    g.byte0 = byte0;
    byte0 += pr[i].N * rowb;
  }
  pl.smem = static_cast<int>(fixed + static_cast<int64_t>(kGsCW) * nslots * slot);
  if (pl.smem > d->max_smem_optin) return BITNET_ERR_UNSUPPORTED;
  return BITNET_OK;
}

template <int MT, int MAXP, int BITS>
cudaError_t run_stream_t(const StreamPlan<MAXP>& pl, cudaStream_t st) {
  auto k = gemv_stream_kernel<MT, MAXP, kGsCW, BITS>;
  cudaError_t e = allow_smem(k, pl.smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(k, dim3(pl.grid), dim3(kGsCW * 32 + 32), pl.smem, st, pl.p);
}

template <int MAXP>
cudaError_t run_stream(const StreamPlan<MAXP>& pl, cudaStream_t st) {
  if (pl.p.bits == 1) return pl.MT == 1 ? run_stream_t<1, MAXP, 1>(pl, st) : cudaErrorInvalidValue;
  if (pl.p.bits == 3) return pl.MT == 1 ? run_stream_t<1, MAXP, 3>(pl, st) : cudaErrorInvalidValue;
  switch (pl.MT) {
    case 1: return run_stream_t<1, MAXP, 2>(pl, st);
    case 2: return run_stream_t<2, MAXP, 2>(pl, st);
    case 4: return run_stream_t<4, MAXP, 2>(pl, st);
    default: return cudaErrorInvalidValue;
  }
}

constexpr int kStreamSmallP = 4;
constexpr int kStreamMaxP = 256;

// ---------------------------------------------------------------------------
// Tensor-core GEMM launch.
// ---------------------------------------------------------------------------
template <int BM, int SS, int AS, int BITS>
cudaError_t run_tc_t(const int8_t* xq, const TcParams& p, cudaStream_t st) {
  CUtensorMap map;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.K), static_cast<cuuint64_t>(p.M)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.K)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcBK), static_cast<cuuint32_t>(BM)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(xq), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto k = tc_gemm_kernel<BM, SS, AS, BITS>;
  constexpr int smem = tc_smem_bytes<BM, SS>();
  cudaError_t e = allow_smem(k, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((p.N + kTcBN - 1) / kTcBN, (p.M + BM - 1) / BM);
  return launch_pdl(k, grid, dim3(kTcThreads), smem, st, map, p);
}

// Persistent tiles of 256 weight rows x BM tokens, one CTA per SM (the
// shared-memory request keeps a second CTA off the SM: both want all 512
// TMEM columns).
template <int BM, int SS, int AS, int BITS>
cudaError_t run_tp_t(const int8_t* xq, const TcParams& p, int sms, cudaStream_t st) {
  static_assert(2 * tp_smem_bytes<BM, SS>() > 233472, "one CTA per SM");
  CUtensorMap map;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.K), static_cast<cuuint64_t>(p.M)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.K)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcBK), static_cast<cuuint32_t>(BM)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(xq), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto k = tc_gemm_persistent_kernel<BM, SS, AS, BITS>;
  constexpr int smem = tp_smem_bytes<BM, SS>();
  cudaError_t e = allow_smem(k, smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = static_cast<int64_t>((p.N + kTpRows - 1) / kTpRows) * ((p.M + BM - 1) / BM);
  const int grid = static_cast<int>(std::min<int64_t>(tiles, sms));
  return launch_pdl(k, dim3(grid), dim3(kTpThreads), smem, st, map, p);
}

// Token tile BM = MMA N.  Up to 64 tokens: one CTA per 128-row tile, 4 TMEM
// A buffers, at most 256 TMEM columns, so two CTAs can share an SM.  Beyond:
// the persistent kernel.
template <int BITS>
cudaError_t run_tc_bits(const int8_t* xq, const TcParams& p, int sms, cudaStream_t st) {
  if (p.M <= 16) return run_tc_t<16, 8, 4, BITS>(xq, p, st);
  if (p.M <= 32) return run_tc_t<32, 8, 4, BITS>(xq, p, st);
  if (p.M <= 64) return run_tc_t<64, 8, 4, BITS>(xq, p, st);
  return run_tp_t<128, 8, 2, BITS>(xq, p, sms, st);
}

cudaError_t run_tc(const int8_t* xq, const TcParams& p, int sms, cudaStream_t st, int bits = 2) {
  return bits == 1 ? run_tc_bits<1>(xq, p, sms, st) : run_tc_bits<2>(xq, p, sms, st);
}

bitnet_status launch_result(cudaError_t e) {
  if (e != cudaSuccess) {
    cudaGetLastError();
    return BITNET_ERR_CUDA;
  }
  e = cudaGetLastError();
  return e == cudaSuccess ? BITNET_OK : BITNET_ERR_CUDA;
}

// Scratch of bitnet_quant_weights_noalloc: the per-block exact-sum bins.
// Every GPU that loads the library holds these 256 KiB until exit.
constexpr int kNoAllocMaxBlocks = 2048;
static __device__ __align__(256) uint64_t g_noalloc_scratch[kNoAllocMaxBlocks * kAbsBins];

// Device address of the scratch array per device, resolved once with that
// device current (the host symbol itself is not a device address).
uint64_t* g_noalloc_ptr[kMaxDevices] = {};

}  // namespace

// ===========================================================================
// Exported C ABI
// ===========================================================================
extern "C" {

size_t bitnet_workspace_bytes(int64_t M, int64_t K, int64_t N) {
  (void)N;
  if (M < 1 || K < 1) return kWsHeader;
  return linear_ws_bytes(M, K);
}

size_t bitnet_quant_weights_workspace_bytes(int64_t N, int64_t K) {
  const int64_t n = N * K;
  int64_t blocks = (n + kAbsMaxPerBlock - 1) / kAbsMaxPerBlock;
  const int64_t want = 148 * 8;
  if (blocks < want) blocks = want;
  return kWsHeader + static_cast<size_t>(blocks) * kAbsBins * sizeof(uint64_t);
}

bitnet_status bitnet_workspace_init(void* ws, size_t ws_bytes, bitnet_stream_t stream) {
  if (ws == nullptr) return BITNET_ERR_NULL;
  if (ws_bytes < kWsHeader || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return BITNET_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, kWsHeader, reinterpret_cast<cudaStream_t>(stream)));
}

bitnet_status bitnet_get_error(void* ws, bitnet_stream_t stream) {
  if (ws == nullptr) return BITNET_ERR_NULL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t h[2] = {0, 0};
  if (cudaMemcpyAsync(h, ws, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return BITNET_ERR_CUDA;
  }
  if (h[0] != 0) {
    if (cudaMemsetAsync(ws, 0, sizeof h, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess) {
      cudaGetLastError();
      return BITNET_ERR_CUDA;
    }
  }
  return static_cast<bitnet_status>(h[0]);
}

const char* bitnet_status_str(bitnet_status s) {
  switch (s) {
    case BITNET_OK: return "ok";
    case BITNET_ERR_NULL: return "null pointer";
    case BITNET_ERR_SHAPE: return "invalid shape (M, N >= 1; K a positive multiple of 16)";
    case BITNET_ERR_ALIGN: return "pointer not 16-byte aligned";
    case BITNET_ERR_DTYPE: return "unknown dtype";
    case BITNET_ERR_UNSUPPORTED: return "unsupported (needs an sm_100 device, or the forced path cannot run)";
    case BITNET_ERR_CUDA: return "CUDA runtime error";
    case BITNET_ERR_TIMEOUT: return "device wait timed out";
    case BITNET_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case BITNET_ERR_VALUE: return "invalid ternary value or code";
  }
  return "unknown status";
}

bitnet_status bitnet_set_wait_limit_us(uint32_t limit_us) {
  if (limit_us == 0) return BITNET_ERR_SHAPE;
  g_limit_ns.store(static_cast<uint64_t>(limit_us) * 1000ull);
  return BITNET_OK;
}

bitnet_status bitnet_quant_weights(const float* W, int64_t N, int64_t K, float eps, int8_t* Wq, float* gamma,
                                   void* ws, size_t ws_bytes, bitnet_stream_t stream) {
  if (W == nullptr || gamma == nullptr || ws == nullptr) return BITNET_ERR_NULL;
  if (check_shape(1, K, N) != BITNET_OK) return BITNET_ERR_SHAPE;
  if (!aligned16(W) || (Wq != nullptr && !aligned16(Wq))) return BITNET_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < bitnet_quant_weights_workspace_bytes(N, K))
    return BITNET_ERR_WORKSPACE;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = N * K;
  int64_t blocks = (n + kAbsMaxPerBlock - 1) / kAbsMaxPerBlock;
  const int64_t want = static_cast<int64_t>(d->sms) * 8;
  if (blocks < want) blocks = want;
  const int64_t cap = static_cast<int64_t>((ws_bytes - kWsHeader) / (kAbsBins * sizeof(uint64_t)));
  if (blocks > cap) blocks = cap;
  int64_t per_block = (n + blocks - 1) / blocks;
  per_block = (per_block + 15) / 16 * 16;          // keep float4 alignment
  if (per_block > kAbsMaxPerBlock) return BITNET_ERR_WORKSPACE;
  blocks = (n + per_block - 1) / per_block;
  uint32_t* status = static_cast<uint32_t*>(ws);
  uint64_t* partial = reinterpret_cast<uint64_t*>(static_cast<uint8_t*>(ws) + kWsHeader);
  absmean_partial_kernel<<<static_cast<unsigned>(blocks), kAbsThreads, 0, st>>>(W, n, per_block, partial, status);
  absmean_finalize_kernel<<<1, kAbsFinThreads, 0, st>>>(partial, static_cast<int>(blocks), n, gamma);
  if (Wq != nullptr) {
    ternarise_kernel<<<elementwise_grid(n / 4, d), 256, 0, st>>>(W, n / 4, gamma, eps, Wq);
  }
  return launch_result(cudaSuccess);
}

bitnet_status bitnet_quant_weights_b1(const float* W, int64_t N, int64_t K, int8_t* Wb, float* beta, void* ws,
                                      size_t ws_bytes, bitnet_stream_t stream) {
  // beta is the absmean of bitnet_quant_weights (same exact sum, same
  // workspace); the signs replace the ternarisation.
  bitnet_status s = bitnet_quant_weights(W, N, K, 0.0f, nullptr, beta, ws, ws_bytes, stream);
  if (s != BITNET_OK || Wb == nullptr) return s;
  if (!aligned16(Wb)) return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  s = device_info(&d);
  if (s != BITNET_OK) return s;
  const int64_t n = N * K;
  binarise_kernel<<<elementwise_grid(n / 4, d), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(W, n / 4, Wb);
  return launch_result(cudaSuccess);
}

bitnet_status bitnet_pack_b1(const int8_t* Wb, int64_t N, int64_t K, uint8_t* Wp, uint32_t* n_invalid,
                             bitnet_stream_t stream) {
  if (Wb == nullptr || Wp == nullptr) return BITNET_ERR_NULL;
  if (check_shape(1, K, N) != BITNET_OK || K % 32 != 0) return BITNET_ERR_SHAPE;
  if (!aligned16(Wb) || !aligned16(Wp)) return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  const int64_t groups = N * K / 32;
  pack_b1_kernel<<<elementwise_grid(groups, d), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      Wb, groups, reinterpret_cast<uint32_t*>(Wp), n_invalid);
  return launch_result(cudaSuccess);
}

bitnet_status bitnet_unpack_b1(const uint8_t* Wp, int64_t N, int64_t K, int8_t* Wb, bitnet_stream_t stream) {
  if (Wb == nullptr || Wp == nullptr) return BITNET_ERR_NULL;
  if (check_shape(1, K, N) != BITNET_OK || K % 32 != 0) return BITNET_ERR_SHAPE;
  if (!aligned16(Wb) || !aligned16(Wp)) return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  const int64_t groups = N * K / 32;
  unpack_b1_kernel<<<elementwise_grid(groups, d), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(Wp), groups, Wb);
  return launch_result(cudaSuccess);
}

bitnet_status bitnet_ternarise(const float* W, int64_t N, int64_t K, const float* gamma, float eps, int8_t* Wq,
                               bitnet_stream_t stream) {
  if (W == nullptr || gamma == nullptr || Wq == nullptr) return BITNET_ERR_NULL;
  if (check_shape(1, K, N) != BITNET_OK) return BITNET_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(Wq)) return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  const int64_t n = N * K;
  ternarise_kernel<<<elementwise_grid(n / 4, d), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(W, n / 4, gamma,
                                                                                                     eps, Wq);
  return launch_result(cudaSuccess);
}

bitnet_status bitnet_pack(const int8_t* Wq, int64_t N, int64_t K, uint8_t* Wp, uint32_t* n_invalid,
                          bitnet_stream_t stream) {
  if (Wq == nullptr || Wp == nullptr) return BITNET_ERR_NULL;
  if (check_shape(1, K, N) != BITNET_OK) return BITNET_ERR_SHAPE;
  if (!aligned16(Wq) || !aligned16(Wp)) return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t groups = N * K / 16;
  pack_kernel<<<elementwise_grid(groups, d), 256, 0, st>>>(Wq, groups, reinterpret_cast<uint32_t*>(Wp), n_invalid);
  stream_fence_kernel<<<1, 32, 0, st>>>();
  return launch_result(cudaSuccess);
}

bitnet_status bitnet_unpack(const uint8_t* Wp, int64_t N, int64_t K, int8_t* Wq, uint32_t* n_invalid,
                            bitnet_stream_t stream) {
  if (Wq == nullptr || Wp == nullptr) return BITNET_ERR_NULL;
  if (check_shape(1, K, N) != BITNET_OK) return BITNET_ERR_SHAPE;
  if (!aligned16(Wq) || !aligned16(Wp)) return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  const int64_t groups = N * K / 16;
  unpack_kernel<<<elementwise_grid(groups, d), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(Wp), groups, Wq, n_invalid);
  return launch_result(cudaSuccess);
}

bitnet_status bitnet_quant_act(const void* x, int x_dtype, int64_t M, int64_t K, const float* rms_gain,
                               float rms_eps, int8_t* xq, float* x_scale, int32_t* x_sum, bitnet_stream_t stream) {
  if (x == nullptr || xq == nullptr || x_scale == nullptr) return BITNET_ERR_NULL;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (check_shape(M, K, 1) != BITNET_OK) return BITNET_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(xq) || (rms_gain != nullptr && !aligned16(rms_gain))) return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  cudaError_t e = launch_pdl(quant_act_kernel, dim3(static_cast<unsigned>(M)), dim3(kActThreads), 0,
                             reinterpret_cast<cudaStream_t>(stream), x, x_dtype, static_cast<int>(K), rms_gain,
                             rms_eps, xq, x_scale, x_sum, static_cast<const void*>(nullptr));
  return launch_result(e);
}

bitnet_status bitnet_quant_act_relu2(const void* gate, const void* up, int x_dtype, int64_t M, int64_t K,
                                     const float* rms_gain, float rms_eps, int8_t* xq, float* x_scale,
                                     int32_t* x_sum, bitnet_stream_t stream) {
  if (gate == nullptr || up == nullptr || xq == nullptr || x_scale == nullptr) return BITNET_ERR_NULL;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (check_shape(M, K, 1) != BITNET_OK) return BITNET_ERR_SHAPE;
  if (!aligned16(gate) || !aligned16(up) || !aligned16(xq) || (rms_gain != nullptr && !aligned16(rms_gain)))
    return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  cudaError_t e = launch_pdl(quant_act_kernel, dim3(static_cast<unsigned>(M)), dim3(kActThreads), 0,
                             reinterpret_cast<cudaStream_t>(stream), gate, x_dtype, static_cast<int>(K), rms_gain,
                             rms_eps, xq, x_scale, x_sum, up);
  return launch_result(e);
}

static bitnet_status linear_impl(const void* x, int x_dtype, const int8_t* xq_in, const float* scale_in,
                                 const int32_t* sum_in, int64_t M, int64_t K, const uint8_t* Wp, int64_t N,
                                 const float* gamma, const float* rms_gain, float rms_eps, void* y, int y_dtype,
                                 int32_t* acc, void* ws, size_t ws_bytes, int path, cudaStream_t st,
                                 const void* x2 = nullptr, const void* resid = nullptr, int bits = 2) {
  if (Wp == nullptr || gamma == nullptr || ws == nullptr) return BITNET_ERR_NULL;
  if (y == nullptr && acc == nullptr) return BITNET_ERR_NULL;
  if (resid != nullptr && y == nullptr) return BITNET_ERR_NULL;
  if ((x2 != nullptr && !aligned16(x2)) || (resid != nullptr && !aligned16(resid))) return BITNET_ERR_ALIGN;
  if (y != nullptr && y_dtype != BITNET_F32 && y_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  bitnet_status s = check_shape(M, K, N);
  if (s != BITNET_OK) return s;
  if (!aligned16(Wp) || (y != nullptr && !aligned16(y)) || (acc != nullptr && !aligned16(acc)) ||
      (rms_gain != nullptr && !aligned16(rms_gain)))
    return BITNET_ERR_ALIGN;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < kWsHeader) return BITNET_ERR_WORKSPACE;
  if (path != BITNET_PATH_AUTO && path != BITNET_PATH_GEMV && path != BITNET_PATH_TC) return BITNET_ERR_UNSUPPORTED;
  DeviceInfo* d;
  s = device_info(&d);
  if (s != BITNET_OK) return s;
  uint32_t* status = static_cast<uint32_t*>(ws);
  const uint64_t limit = g_limit_ns.load();

  GemvPlan gp;
  bool gemv_ok = plan_gemv(d, M, K, N, gp) == BITNET_OK;
  // the gated input and the residual are in the streaming GEMV (K % 64 == 0)
  // and the tensor-core path, not in the padded-row GEMV
  if ((x2 != nullptr || resid != nullptr) && K % 64 != 0) gemv_ok = false;
  // 1-bit signs: the streaming GEMV for one token, the tensor-core path otherwise
  if (bits == 1) {
    if (K % 128 != 0) return BITNET_ERR_SHAPE;
    gemv_ok = (M == 1 && x != nullptr);
  }
  // base-3: one token through the streaming GEMV only (a decode format)
  if (bits == 3) {
    if (M != 1 || x == nullptr) return BITNET_ERR_UNSUPPORTED;
    gemv_ok = true;
  }
  if (path == BITNET_PATH_GEMV && !gemv_ok) return BITNET_ERR_UNSUPPORTED;
  const bool use_gemv = (path == BITNET_PATH_GEMV) || (path == BITNET_PATH_AUTO && gemv_ok);

  if (use_gemv && (K % 64 == 0 || bits == 3)) {
    StreamProblem sp{x != nullptr ? x : static_cast<const void*>(xq_in), Wp, gamma, rms_gain, scale_in, y, acc, K, N,
                     x2, resid};
    auto* pl = new (std::nothrow) StreamPlan<kStreamSmallP>;
    if (pl == nullptr) return BITNET_ERR_CUDA;
    s = plan_stream<kStreamSmallP>(d, &sp, 1, M, x != nullptr ? x_dtype : BITNET_F32, x == nullptr, rms_eps,
                                   y != nullptr ? y_dtype : BITNET_F32, *pl, bits);
    if (s == BITNET_OK) {
      pl->p.limit_ns = limit;
      pl->p.status = status;
    }
    cudaError_t e = (s == BITNET_OK) ? run_stream<kStreamSmallP>(*pl, st) : cudaSuccess;
    delete pl;
    // A very long row (the activations plus one packed row per ring slot
    // beyond shared memory) has no streaming plan; the automatic choice then
    // takes the tensor-core path, which handles any K.  Base-3 weights have
    // no tensor-core path.
    const bool to_tc = s == BITNET_ERR_UNSUPPORTED && path == BITNET_PATH_AUTO && bits != 3;
    if (!to_tc) {
      if (s != BITNET_OK) return s;
      return launch_result(e);
    }
  } else if (use_gemv) {
    GemvParams& p = gp.p;
    p.x = x;
    p.x_dtype = x_dtype;
    p.gain = rms_gain;
    p.rms_eps = rms_eps;
    p.xq = xq_in;
    p.x_scale = scale_in;
    p.Wp = Wp;
    p.gamma = gamma;
    p.y = y;
    p.y_dtype = y_dtype;
    p.acc = acc;
    p.limit_ns = limit;
    p.status = status;
    cudaError_t e = (x != nullptr) ? run_gemv<true>(gp, st) : run_gemv<false>(gp, st);
    return launch_result(e);
  }

  // Tensor-core path: quantised activations must sit in memory for TMA.
  s = get_encoder();
  if (s != BITNET_OK) return s;
  const int8_t* xq = xq_in;
  const float* scale = scale_in;
  const int32_t* sum = sum_in;
  if (x != nullptr) {
    if (ws_bytes < linear_ws_bytes(M, K)) return BITNET_ERR_WORKSPACE;
    LinearWs w = carve(ws, M, K);
    cudaError_t e = launch_pdl(quant_act_kernel, dim3(static_cast<unsigned>(M)), dim3(kActThreads), 0, st, x,
                               x_dtype, static_cast<int>(K), rms_gain, rms_eps, w.xq, w.scale, w.sum, x2);
    if (e != cudaSuccess) return launch_result(e);
    xq = w.xq;
    scale = w.scale;
    sum = w.sum;
  } else if (sum == nullptr) {
    if (ws_bytes < linear_ws_bytes(M, K)) return BITNET_ERR_WORKSPACE;
    LinearWs w = carve(ws, M, K);
    cudaError_t e = launch_pdl(xq_rowsum_kernel, dim3(static_cast<unsigned>(M)), dim3(kActThreads), 0, st, xq,
                               static_cast<int>(K), w.sum);
    if (e != cudaSuccess) return launch_result(e);
    sum = w.sum;
  }
  TcParams p;
  p.Wp = Wp;
  p.resid = resid;
  p.gamma = gamma;
  p.x_scale = scale;
  p.x_sum = sum;
  p.y = y;
  p.y_dtype = y_dtype;
  p.acc = acc;
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.N = static_cast<int>(N);
  p.KB = static_cast<int>((K + kTcBK - 1) / kTcBK);
  p.wvec = (K % 64 == 0) ? 1 : 0;
  p.limit_ns = limit;
  p.status = status;
  return launch_result(run_tc(xq, p, d->sms, st, bits));
}

bitnet_status bitnet_linear_ex(const void* x, int x_dtype, int64_t M, int64_t K, const uint8_t* Wp, int64_t N,
                               const float* gamma, const float* rms_gain, float rms_eps, void* y, int y_dtype,
                               void* ws, size_t ws_bytes, int path, bitnet_stream_t stream) {
  if (x == nullptr || y == nullptr) return BITNET_ERR_NULL;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (!aligned16(x)) return BITNET_ERR_ALIGN;
  return linear_impl(x, x_dtype, nullptr, nullptr, nullptr, M, K, Wp, N, gamma, rms_gain, rms_eps, y, y_dtype,
                     nullptr, ws, ws_bytes, path, reinterpret_cast<cudaStream_t>(stream));
}

bitnet_status bitnet_linear(const void* x, int x_dtype, int64_t M, int64_t K, const uint8_t* Wp, int64_t N,
                            const float* gamma, const float* rms_gain, float rms_eps, void* y, int y_dtype, void* ws,
                            size_t ws_bytes, bitnet_stream_t stream) {
  return bitnet_linear_ex(x, x_dtype, M, K, Wp, N, gamma, rms_gain, rms_eps, y, y_dtype, ws, ws_bytes,
                          BITNET_PATH_AUTO, stream);
}

bitnet_status bitnet_linear_relu2(const void* gate, const void* up, int x_dtype, int64_t M, int64_t K,
                                  const uint8_t* Wp, int64_t N, const float* gamma, const float* rms_gain,
                                  float rms_eps, const void* resid, void* y, int y_dtype, void* ws, size_t ws_bytes,
                                  bitnet_stream_t stream) {
  if (gate == nullptr || up == nullptr || y == nullptr) return BITNET_ERR_NULL;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (!aligned16(gate)) return BITNET_ERR_ALIGN;
  return linear_impl(gate, x_dtype, nullptr, nullptr, nullptr, M, K, Wp, N, gamma, rms_gain, rms_eps, y, y_dtype,
                     nullptr, ws, ws_bytes, BITNET_PATH_AUTO, reinterpret_cast<cudaStream_t>(stream), up, resid);
}

bitnet_status bitnet_linear_b1(const void* x, int x_dtype, int64_t M, int64_t K, const uint8_t* Wp, int64_t N,
                               const float* beta, const float* rms_gain, float rms_eps, void* y, int y_dtype,
                               void* ws, size_t ws_bytes, bitnet_stream_t stream) {
  if (x == nullptr || y == nullptr) return BITNET_ERR_NULL;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (!aligned16(x)) return BITNET_ERR_ALIGN;
  return linear_impl(x, x_dtype, nullptr, nullptr, nullptr, M, K, Wp, N, beta, rms_gain, rms_eps, y, y_dtype,
                     nullptr, ws, ws_bytes, BITNET_PATH_AUTO, reinterpret_cast<cudaStream_t>(stream), nullptr,
                     nullptr, 1);
}

bitnet_status bitnet_linear_q(const int8_t* xq, const float* x_scale, const int32_t* x_sum, int64_t M, int64_t K,
                              const uint8_t* Wp, int64_t N, const float* gamma, void* y, int y_dtype, int32_t* acc,
                              void* ws, size_t ws_bytes, int path, bitnet_stream_t stream) {
  if (xq == nullptr || x_scale == nullptr) return BITNET_ERR_NULL;
  if (!aligned16(xq)) return BITNET_ERR_ALIGN;
  return linear_impl(nullptr, BITNET_F32, xq, x_scale, x_sum, M, K, Wp, N, gamma, nullptr, 0.0f, y, y_dtype, acc, ws,
                     ws_bytes, path, reinterpret_cast<cudaStream_t>(stream));
}

static bitnet_status grouped_impl(const bitnet_gemv_problem* problems, int count, int64_t M, int x_dtype,
                                  float rms_eps, int y_dtype, void* ws, size_t ws_bytes, bitnet_stream_t stream,
                                  int bits) {
  if (problems == nullptr || ws == nullptr) return BITNET_ERR_NULL;
  if (count < 1 || count > kStreamMaxP) return BITNET_ERR_SHAPE;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (y_dtype != BITNET_F32 && y_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (M < 1 || M > (bits != 2 ? 1 : kGemvMaxM)) return BITNET_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < kWsHeader) return BITNET_ERR_WORKSPACE;
  std::vector<StreamProblem> sp(count);
  for (int i = 0; i < count; ++i) {
    const bitnet_gemv_problem& q = problems[i];
    if (q.x == nullptr || q.Wp == nullptr || q.gamma == nullptr || q.y == nullptr) return BITNET_ERR_NULL;
    bitnet_status s = check_shape(M, q.K, q.N);
    if (s != BITNET_OK) return s;
    if ((bits == 2 && q.K % 64 != 0) || (bits == 1 && q.K % 128 != 0)) return BITNET_ERR_SHAPE;
    if (!aligned16(q.x) || !aligned16(q.Wp) || !aligned16(q.y) || (q.rms_gain != nullptr && !aligned16(q.rms_gain)))
      return BITNET_ERR_ALIGN;
    sp[i] = StreamProblem{q.x, q.Wp, q.gamma, q.rms_gain, nullptr, q.y, nullptr, q.K, q.N};
  }
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const uint64_t limit = g_limit_ns.load();
  if (count <= kStreamSmallP) {
    auto* pl = new (std::nothrow) StreamPlan<kStreamSmallP>;
    if (pl == nullptr) return BITNET_ERR_CUDA;
    s = plan_stream<kStreamSmallP>(d, sp.data(), count, M, x_dtype, false, rms_eps, y_dtype, *pl, bits);
    cudaError_t e = cudaSuccess;
    if (s == BITNET_OK) {
      pl->p.limit_ns = limit;
      pl->p.status = static_cast<uint32_t*>(ws);
      e = run_stream<kStreamSmallP>(*pl, st);
    }
    delete pl;
    return s != BITNET_OK ? s : launch_result(e);
  }
  auto* pl = new (std::nothrow) StreamPlan<kStreamMaxP>;
  if (pl == nullptr) return BITNET_ERR_CUDA;
  s = plan_stream<kStreamMaxP>(d, sp.data(), count, M, x_dtype, false, rms_eps, y_dtype, *pl, bits);
  cudaError_t e = cudaSuccess;
  if (s == BITNET_OK) {
    pl->p.limit_ns = limit;
    pl->p.status = static_cast<uint32_t*>(ws);
    e = run_stream<kStreamMaxP>(*pl, st);
  }
  delete pl;
  return s != BITNET_OK ? s : launch_result(e);
}

bitnet_status bitnet_linear_grouped(const bitnet_gemv_problem* problems, int count, int64_t M, int x_dtype,
                                    float rms_eps, int y_dtype, void* ws, size_t ws_bytes, bitnet_stream_t stream) {
  return grouped_impl(problems, count, M, x_dtype, rms_eps, y_dtype, ws, ws_bytes, stream, 2);
}

bitnet_status bitnet_linear_grouped_b1(const bitnet_gemv_problem* problems, int count, int x_dtype, float rms_eps,
                                       int y_dtype, void* ws, size_t ws_bytes, bitnet_stream_t stream) {
  return grouped_impl(problems, count, 1, x_dtype, rms_eps, y_dtype, ws, ws_bytes, stream, 1);
}

bitnet_status bitnet_linear_grouped_t3(const bitnet_gemv_problem* problems, int count, int x_dtype, float rms_eps,
                                       int y_dtype, void* ws, size_t ws_bytes, bitnet_stream_t stream) {
  return grouped_impl(problems, count, 1, x_dtype, rms_eps, y_dtype, ws, ws_bytes, stream, 3);
}

int64_t bitnet_t3_row_bytes(int64_t K) { return K < 1 ? 0 : gs_row_bytes(K, 3); }

bitnet_status bitnet_pack_t3(const int8_t* Wq, int64_t N, int64_t K, uint8_t* Wp, uint32_t* n_invalid,
                             bitnet_stream_t stream) {
  if (Wq == nullptr || Wp == nullptr) return BITNET_ERR_NULL;
  if (check_shape(1, K, N) != BITNET_OK) return BITNET_ERR_SHAPE;
  if (!aligned16(Wp)) return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  const int64_t rb = gs_row_bytes(K, 3);
  pack_t3_kernel<<<elementwise_grid(N * rb / 4, d), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      Wq, N, K, rb, reinterpret_cast<uint32_t*>(Wp), n_invalid);
  return launch_result(cudaSuccess);
}

bitnet_status bitnet_unpack_t3(const uint8_t* Wp, int64_t N, int64_t K, int8_t* Wq, uint32_t* n_invalid,
                               bitnet_stream_t stream) {
  if (Wq == nullptr || Wp == nullptr) return BITNET_ERR_NULL;
  if (check_shape(1, K, N) != BITNET_OK) return BITNET_ERR_SHAPE;
  if (!aligned16(Wp)) return BITNET_ERR_ALIGN;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  const int64_t rb = gs_row_bytes(K, 3);
  unpack_t3_kernel<<<elementwise_grid(N * rb / 4, d), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(Wp), N, K, rb, Wq, n_invalid);
  return launch_result(cudaSuccess);
}

bitnet_status bitnet_linear_t3(const void* x, int x_dtype, int64_t K, const uint8_t* Wp, int64_t N,
                               const float* gamma, const float* rms_gain, float rms_eps, void* y, int y_dtype,
                               void* ws, size_t ws_bytes, bitnet_stream_t stream) {
  if (x == nullptr || y == nullptr) return BITNET_ERR_NULL;
  if (x_dtype != BITNET_F32 && x_dtype != BITNET_BF16) return BITNET_ERR_DTYPE;
  if (!aligned16(x)) return BITNET_ERR_ALIGN;
  return linear_impl(x, x_dtype, nullptr, nullptr, nullptr, 1, K, Wp, N, gamma, rms_gain, rms_eps, y, y_dtype,
                     nullptr, ws, ws_bytes, BITNET_PATH_AUTO, reinterpret_cast<cudaStream_t>(stream), nullptr,
                     nullptr, 3);
}

bitnet_status bitnet_watchdog_selftest(void* ws, size_t ws_bytes, uint32_t limit_us, bitnet_stream_t stream) {
  if (ws == nullptr) return BITNET_ERR_NULL;
  if (ws_bytes < kWsHeader || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return BITNET_ERR_WORKSPACE;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  watchdog_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull, static_cast<uint32_t*>(ws));
  return launch_result(cudaSuccess);
}

// The streaming GEMV's plan for a described device, without touching one.
bitnet_status bitnet_debug_stream_plan(const int64_t* K, const int64_t* N, int count, int64_t M, int bits,
                                       int prequant, int sms, int smem_optin, int64_t* shape, int32_t* rows,
                                       int32_t* task) {
  if (K == nullptr || N == nullptr) return BITNET_ERR_NULL;
  if (count < 1 || count > kStreamMaxP || sms < 1 || smem_optin < 1) return BITNET_ERR_SHAPE;
  if (bits != 1 && bits != 2 && bits != 3) return BITNET_ERR_UNSUPPORTED;
  std::vector<StreamProblem> sp(count);
  for (int i = 0; i < count; ++i) {
    bitnet_status s = check_shape(M, K[i], N[i]);
    if (s != BITNET_OK) return s;
    sp[i] = StreamProblem{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, K[i], N[i]};
  }
  DeviceInfo d;
  d.init = true;
  d.ok = true;
  d.sms = sms;
  d.max_smem_optin = smem_optin;
  auto* pl = new (std::nothrow) StreamPlan<kStreamMaxP>;
  if (pl == nullptr) return BITNET_ERR_CUDA;
  const bitnet_status s = plan_stream<kStreamMaxP>(&d, sp.data(), count, M, BITNET_BF16, prequant != 0, 1e-5f,
                                                   BITNET_BF16, *pl, bits);
  if (s == BITNET_OK) {
    if (shape != nullptr) {
      shape[0] = pl->grid;
      shape[1] = pl->smem;
      shape[2] = pl->p.nxb;
      shape[3] = pl->p.nslots;
      shape[4] = pl->p.slot_bytes;
    }
    for (int i = 0; i < count; ++i) {
      if (rows != nullptr) rows[i] = pl->p.prob[i].rc;
      if (task != nullptr) task[i] = pl->p.prob[i].task;
    }
  }
  delete pl;
  return s;
}

// Variant of bitnet_quant_weights that allocates nothing: its scratch is the
// file-scope array above instead of a caller workspace.
bitnet_status bitnet_quant_weights_noalloc(const float* W, int64_t N, int64_t K, float eps, int8_t* Wq,
                                           float* gamma, bitnet_stream_t stream) {
  if (W == nullptr || gamma == nullptr) return BITNET_ERR_NULL;
  if (check_shape(1, K, N) != BITNET_OK) return BITNET_ERR_SHAPE;
  if (!aligned16(W) || (Wq != nullptr && !aligned16(Wq))) return BITNET_ERR_ALIGN;
  // the scratch holds kNoAllocMaxBlocks blocks of at most kAbsMaxPerBlock elements
  if (N * K > static_cast<int64_t>(kNoAllocMaxBlocks) * kAbsMaxPerBlock) return BITNET_ERR_SHAPE;
  DeviceInfo* d;
  bitnet_status s = device_info(&d);
  if (s != BITNET_OK) return s;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return BITNET_ERR_CUDA;
  }
  uint64_t* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
        cudaGetLastError();
        return BITNET_ERR_CUDA;
      }
      g_noalloc_ptr[dev] = static_cast<uint64_t*>(ptr);
    }
    scratch = g_noalloc_ptr[dev];
  }
  const int64_t n = N * K;
  // same partition rule as bitnet_quant_weights, capped by the scratch size
  int64_t blocks = (n + kAbsMaxPerBlock - 1) / kAbsMaxPerBlock;
  const int64_t want = static_cast<int64_t>(d->sms) * 8;
  if (blocks < want) blocks = want;
  if (blocks > kNoAllocMaxBlocks) blocks = kNoAllocMaxBlocks;
  int64_t per_block = (n + blocks - 1) / blocks;
  per_block = (per_block + 15) / 16 * 16;   // <= kAbsMaxPerBlock by the size check above
  blocks = (n + per_block - 1) / per_block;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  absmean_partial_kernel<<<static_cast<unsigned>(blocks), kAbsThreads, 0, st>>>(W, n, per_block, scratch, nullptr);
  absmean_finalize_kernel<<<1, kAbsFinThreads, 0, st>>>(scratch, static_cast<int>(blocks), n, gamma);
  if (Wq != nullptr) {
    ternarise_kernel<<<elementwise_grid(n / 4, d), 256, 0, st>>>(W, n / 4, gamma, eps, Wq);
  }
  return launch_result(cudaSuccess);
}

}  // extern "C"

