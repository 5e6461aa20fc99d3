// libmla: the C-ABI entry points declared in include/mla.h.
//
// Host side only: argument validation, TMA tensor-map encoding (through the
// driver entry point, so the library needs no -lcuda), launch configuration
// and status mapping.  Every step of the computation runs in the kernels
// included below; there is no host fallback.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "mla.h"
#include "dense_fwd.cuh"
#include "merge.cuh"
#include "sparse_fwd.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 4000000000ull;  // 4 s per barrier wait

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

uint64_t wait_timeout_ns() {
  static uint64_t t = []() -> uint64_t {
    const char* e = std::getenv("MLA_WAIT_TIMEOUT_MS");
    if (e != nullptr) {
      const long long ms = std::atoll(e);
      if (ms > 0 && ms < 600000) return static_cast<uint64_t>(ms) * 1000000ull;
    }
    return kDefaultTimeoutNs;
  }();
  return t;
}

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context, or 0 when there is
// none (or the driver cannot say).  A device's primary context is created
// anew after cudaDeviceReset or after it was released, and what was set up
// in the old one (kernel attributes, device addresses of module variables)
// does not carry over, so the per-device state below is keyed on this id.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext c = nullptr;
  if (get_cur == nullptr || get_id == nullptr || get_cur(&c) != CUDA_SUCCESS || c == nullptr)
    return 0;
  unsigned long long id = 0;
  return get_id(c, &id) == CUDA_SUCCESS ? id : 0;
}

// Per-device state, set up once per CUDA context: architecture check, kernel
// attributes and launch sizes.  `ctx` is published last (release) and read
// first (acquire), so a thread that sees its own context id there also sees
// the fields written before it.
struct DeviceState {
  std::atomic<unsigned long long> ctx{0};  // context the fields belong to (0: none)
  std::atomic<int> status{MLA_OK};         // MLA_OK or MLA_ERR_UNSUPPORTED
  std::atomic<int> sms{0};
  std::atomic<int> dense_clusters{0};      // co-resident 2-CTA clusters of the dense kernel
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

// The set-up itself (with the device's context current).
int setup_device(int dev, int* status, int* sms, int* clusters) {
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (major != 10 || minor != 0) {
    *status = MLA_ERR_UNSUPPORTED;
    return MLA_OK;
  }
  {
    // Every qk width's kernel: its shared memory, and the launch register
    // count its setmaxnreg split assumes (a different count could make the
    // warps that grow wait for ever).
    const void* kernels[3] = {reinterpret_cast<const void*>(mla::dense::dense_fwd_kernel<128>),
                              reinterpret_cast<const void*>(mla::dense::dense_fwd_kernel<192>),
                              reinterpret_cast<const void*>(mla::dense::dense_fwd_kernel<256>)};
    const int smem[3] = {mla::dense::Geo<128>::kSmemBytes, mla::dense::Geo<192>::kSmemBytes,
                         mla::dense::Geo<256>::kSmemBytes};
    for (int i = 0; i < 3; ++i) {
      if (cudaFuncSetAttribute(kernels[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem[i]) != cudaSuccess)
        return MLA_ERR_CUDA;
      cudaFuncAttributes fa;
      if (cudaFuncGetAttributes(&fa, kernels[i]) != cudaSuccess) return MLA_ERR_CUDA;
      if (fa.numRegs != mla::dense::kLaunchRegs) {
        *status = MLA_ERR_UNSUPPORTED;
        return MLA_OK;
      }
    }
  }
  if (cudaFuncSetAttribute(mla::sparse::sparse_fwd_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           mla::sparse::kSmemBytes) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (encode_fn() == nullptr) return MLA_ERR_CUDA;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return MLA_ERR_CUDA;
  {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (*sms / 2), 1, 1);
    cfg.blockDim = dim3(mla::dense::kThreads, 1, 1);
    cfg.dynamicSmemBytes = mla::dense::Geo<256>::kSmemBytes;  // the largest of the three
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(clusters, mla::dense::dense_fwd_kernel<256>, &cfg) !=
            cudaSuccess ||
        *clusters < 1)
      return MLA_ERR_CUDA;
  }
  *status = MLA_OK;
  return MLA_OK;
}

// Checks the current device and sets it up in its current context (once per
// context).  On success *dev_out is the device.
int prepare_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  *dev_out = dev;
  DeviceState& d = g_dev[dev];
  unsigned long long ctx = current_context_id();
  if (ctx != 0 && d.ctx.load(std::memory_order_acquire) == ctx)
    return d.status.load(std::memory_order_relaxed);
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (ctx == 0) {
    // No context is current yet: the runtime creates the device's primary
    // context lazily; cudaSetDevice makes it current now.
    if (cudaSetDevice(dev) != cudaSuccess) return MLA_ERR_CUDA;
    ctx = current_context_id();
  }
  if (ctx != 0 && d.ctx.load(std::memory_order_relaxed) == ctx)
    return d.status.load(std::memory_order_relaxed);
  int status = MLA_OK, sms = 0, clusters = 0;
  const int st = setup_device(dev, &status, &sms, &clusters);
  if (st != MLA_OK) return st;
  d.status.store(status, std::memory_order_relaxed);
  d.sms.store(sms, std::memory_order_relaxed);
  d.dense_clusters.store(clusters, std::memory_order_relaxed);
  d.ctx.store(ctx, std::memory_order_release);  // 0 (unknown context): set up again next call
  return status;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 2-D bf16 tensor map over a row-major [rows, cols] matrix with a
// 64-column x box_rows box and the 128-byte swizzle.  Rows past `rows` read
// as zero.
int encode_rows(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                uint32_t box_rows) {
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
                                 dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_CUDA;
}

// 3-D bf16 tensor map over [rows, heads, dim] with arbitrary row and head
// strides (elements; the dim is contiguous), a 64-element x 1-head x
// box_rows box and the 128-byte swizzle.  Rows past `rows` read as zero.
int encode_heads(CUtensorMap* map, const void* base, uint64_t dim, uint64_t heads, uint64_t rows,
                 int64_t head_stride, int64_t row_stride, uint32_t box_rows) {
  const cuuint64_t dims[3] = {dim, heads, rows};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_stride) * 2,
                                 static_cast<cuuint64_t>(row_stride) * 2};
  const cuuint32_t box[3] = {64, 1, box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                                 dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MLA_OK : MLA_ERR_INVALID_ARG;
}

// Strides a TMA map accepts: positive, a multiple of 8 elements (16 bytes)
// and below 2^39 elements.
bool good_stride(int64_t st) { return st > 0 && st % 8 == 0 && st < (int64_t{1} << 39); }

int launch_status() { return cudaGetLastError() == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// Scratch for mla_prefill_fwd_noalloc: the dense kernels' work list for
// callers that cannot allocate.  In host code `g_noalloc_scratch` is only a
// stand-in symbol; the device address comes from cudaGetSymbolAddress, with
// the device current, once per device and CUDA context (a context created
// anew, e.g. after cudaDeviceReset, may place the array elsewhere), and is
// cached here.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_NOALLOC_SCRATCH_BYTES];
struct NoallocScratch {
  unsigned long long ctx = 0;  // context `ptr` belongs to (0: none)
  void* ptr = nullptr;
};
NoallocScratch g_noalloc[kMaxDevices];  // guarded by g_noalloc_mu
std::mutex g_noalloc_mu;

// Device address of the scratch array in the current context of `dev`
// (prepare_device has made that context current).  The cache is read and
// written under one mutex, so the context id and the address always belong
// together, also when several contexts of a device are used from different
// threads; a context id of 0 (not known) is never cached.
int noalloc_scratch(int dev, void** out) {
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocScratch& n = g_noalloc[dev];
  if (ctx != 0 && n.ctx == ctx) {
    *out = n.ptr;
    return MLA_OK;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  n.ptr = p;
  n.ctx = ctx;
  *out = p;
  return MLA_OK;
}

__global__ void wait_timeout_probe(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mla::mbar_init(mla::smem_u32(&bar), 1);
    abort_flag = 0;
    mla::fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must give up after limit_ns.
  mla::mbar_wait(mla::smem_u32(&bar), 0, &abort_flag, MLA_DEVSTAT_WAIT_TIMEOUT_TEST, limit_ns);
  __syncthreads();
}

}  // namespace

extern "C" {

const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK:
      return "MLA_OK";
    case MLA_ERR_INVALID_ARG:
      return "MLA_ERR_INVALID_ARG: invalid argument (null/misaligned pointer or bad size)";
    case MLA_ERR_UNSUPPORTED:
      return "MLA_ERR_UNSUPPORTED: needs an sm_100 (B200) GPU and the supported shapes";
    case MLA_ERR_CUDA:
      return "MLA_ERR_CUDA: a CUDA call or kernel launch failed";
    case MLA_ERR_SCRATCH_TOO_SMALL:
      return "MLA_ERR_SCRATCH_TOO_SMALL: the call needs more work-list space than the fixed "
             "scratch of mla_prefill_fwd_noalloc (use mla_prefill_fwd with a workspace)";
    default:
      return "unknown mla_status";
  }
}

int mla_version(void) { return 100; }

size_t mla_prefill_workspace_size(int batch, int total_q) {
  if (batch < 1 || total_q < 0) return 0;
  const size_t entries =
      (static_cast<size_t>(total_q) + mla::dense::kTileRows - 1) / mla::dense::kTileRows +
      static_cast<size_t>(batch);
  return mla::dense::kWsHeaderBytes + entries * sizeof(int2);
}

}  // extern "C"

namespace {

// One dense prefill call: the arguments of every dense entry point.  The
// context (k_ctx, v_ctx, cu_ctx), the sinks and the output scale are
// optional (null).
struct DenseCall {
  const void* q;
  int64_t q_rs, q_hs;
  const void* k;
  int64_t k_rs, k_hs;
  const void* v;
  int64_t v_rs, v_hs;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const void* k_ctx = nullptr;
  const void* v_ctx = nullptr;
  const int32_t* cu_ctx = nullptr;
  int max_ctx = 0, total_ctx = 0;
  const float* sinks = nullptr;
  const float* out_scale = nullptr;
  int nsplit = 1;  // split-KV: the partials live in the workspace after the work list
  int qk_dim = mla::dense::kDqk;  // 128, 192 or 256
  long long out_rs = 0, out_hs = 0;  // output strides in elements (0: packed [T, H, 128])
  int max_q, max_k;
  float scale;
  int causal;
  void* out;
  float* lse;
  mla_stream_t stream;
  int batch, num_heads, total_q, total_k;
  void* workspace;
  size_t workspace_bytes;
};

// Split-KV partials follow the work list, 256-byte aligned.
size_t splitkv_parts_offset(size_t work_list_bytes) { return (work_list_bytes + 255) & ~size_t{255}; }

int dense_call(const DenseCall& c) {
  using namespace mla::dense;
  if (c.q == nullptr || c.k == nullptr || c.v == nullptr || c.cu_q == nullptr ||
      c.cu_k == nullptr || c.out == nullptr || c.workspace == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(c.q, 16) || !aligned(c.k, 16) || !aligned(c.v, 16) || !aligned(c.out, 16) ||
      !aligned(c.workspace, 16) || !aligned(c.cu_q, 4) || !aligned(c.cu_k, 4) ||
      (c.lse && !aligned(c.lse, 4)) || (c.sinks && !aligned(c.sinks, 4)) ||
      (c.out_scale && !aligned(c.out_scale, 4)))
    return MLA_ERR_INVALID_ARG;
  if (c.batch < 1 || c.num_heads < 1 || c.num_heads > 65535 || c.total_q < 0 || c.total_k < 0 ||
      c.max_q < 0 || c.max_k < 0 || (c.causal != 0 && c.causal != 1))
    return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(c.scale) || !(c.scale > 0.0f)) return MLA_ERR_INVALID_ARG;
  if (c.qk_dim != 128 && c.qk_dim != 192 && c.qk_dim != 256) return MLA_ERR_INVALID_ARG;
  if (!good_stride(c.q_rs) || !good_stride(c.q_hs) || !good_stride(c.k_rs) ||
      !good_stride(c.k_hs) || !good_stride(c.v_rs) || !good_stride(c.v_hs))
    return MLA_ERR_INVALID_ARG;
  const bool ctx = c.cu_ctx != nullptr || c.k_ctx != nullptr || c.v_ctx != nullptr;
  if (ctx && (c.cu_ctx == nullptr || c.k_ctx == nullptr || c.v_ctx == nullptr ||
              !aligned(c.k_ctx, 16) || !aligned(c.v_ctx, 16) || !aligned(c.cu_ctx, 4) ||
              c.total_ctx < 0 || c.max_ctx < 0))
    return MLA_ERR_INVALID_ARG;
  if (c.nsplit < 1 || c.nsplit > MLA_MAX_SPLITS || (c.nsplit > 1 && (ctx || c.sinks || c.out_scale)))
    return MLA_ERR_INVALID_ARG;
  const size_t need = mla_prefill_workspace_size(c.batch, c.total_q);
  const size_t need_all =
      c.nsplit > 1 ? mla_prefill_splitkv_workspace_size(c.batch, c.total_q, c.num_heads, c.nsplit)
                   : need;
  if (need_all == 0 || c.workspace_bytes < need_all) return MLA_ERR_INVALID_ARG;
  // the kernels count tiles (work-list entries x heads x splits, plus one
  // grab per cluster past the end) in int
  if (static_cast<long long>((need - kWsHeaderBytes) / sizeof(int2)) * c.num_heads * c.nsplit >
      INT32_MAX - 65536)
    return MLA_ERR_INVALID_ARG;
  int dev = 0;
  int st = prepare_device(&dev);
  if (st != MLA_OK) return st;
  if (c.total_q == 0) return MLA_OK;  // nothing to compute

  CUtensorMap tq, tk, tv, tkc, tvc;
  const uint64_t kv_rows = c.total_k > 0 ? static_cast<uint64_t>(c.total_k) : 1;
  const uint64_t H = static_cast<uint64_t>(c.num_heads);
  const uint64_t dqk = static_cast<uint64_t>(c.qk_dim);
  if ((st = encode_heads(&tq, c.q, dqk, H, static_cast<uint64_t>(c.total_q), c.q_hs, c.q_rs,
                         kCtaRows)) != MLA_OK ||
      (st = encode_heads(&tk, c.k, dqk, H, kv_rows, c.k_hs, c.k_rs, kHalfKeys)) != MLA_OK ||
      (st = encode_heads(&tv, c.v, kDv, H, kv_rows, c.v_hs, c.v_rs, 64)) != MLA_OK)
    return st;
  if (ctx) {
    // the context is packed: [total_ctx, H, 192] and [total_ctx, H, 128]
    const uint64_t c_rows = c.total_ctx > 0 ? static_cast<uint64_t>(c.total_ctx) : 1;
    const int64_t hs = c.num_heads;
    if ((st = encode_heads(&tkc, c.k_ctx, dqk, H, c_rows, c.qk_dim, hs * c.qk_dim, kHalfKeys)) !=
            MLA_OK ||
        (st = encode_heads(&tvc, c.v_ctx, kDv, H, c_rows, kDv, hs * kDv, 64)) != MLA_OK)
      return st;
  } else {
    tkc = tk;  // not read: every sequence has an empty context
    tvc = tv;
  }

  const cudaStream_t s = reinterpret_cast<cudaStream_t>(c.stream);
  WsHeader* ws = static_cast<WsHeader*>(c.workspace);
  int2* entries = reinterpret_cast<int2*>(static_cast<char*>(c.workspace) + kWsHeaderBytes);
  const int capacity = static_cast<int>((need - kWsHeaderBytes) / sizeof(int2));
  dense_plan_kernel<<<1, kPlanThreads, 0, s>>>(c.cu_q, c.cu_k, c.cu_ctx, c.batch, c.causal, ws,
                                               entries, capacity, c.num_heads, c.nsplit);
  if ((st = launch_status()) != MLA_OK) return st;

  Params p;
  p.cu_q = c.cu_q;
  p.cu_k = c.cu_k;
  p.cu_ctx = c.cu_ctx;
  p.out = c.out;
  p.out_rs = c.out_rs != 0 ? c.out_rs : static_cast<long long>(c.num_heads) * kDv;
  p.out_hs = c.out_hs != 0 ? c.out_hs : kDv;
  p.lse = c.lse;
  p.sinks = c.sinks;
  p.out_scale = c.out_scale;
  p.nsplit = c.nsplit;
  p.o_part = nullptr;
  p.lse_part = nullptr;
  if (c.nsplit > 1) {
    char* part = static_cast<char*>(c.workspace) + splitkv_parts_offset(need);
    p.o_part = reinterpret_cast<float*>(part);
    p.lse_part = reinterpret_cast<float*>(
        part + static_cast<size_t>(c.nsplit) * c.total_q * c.num_heads * kDv * sizeof(float));
  }
  // 32-byte stores where every output row starts on a 32-byte boundary: the
  // base, and the row and head strides in bytes (bf16 or e4m3 elements);
  // the partials' rows are 512 bytes.
  {
    const long long esz = c.out_scale != nullptr ? 1 : 2;
    const bool out32 = aligned(c.out, 32) && (p.out_rs * esz) % 32 == 0 &&
                       (p.out_hs * esz) % 32 == 0;
    p.wide_out = (out32 ? 1 : 0) | (p.o_part != nullptr && aligned(p.o_part, 32) ? 2 : 0);
  }
  p.ws = ws;
  p.entries = entries;
  p.num_heads = c.num_heads;
  p.total_q = c.total_q;
  p.causal = c.causal;
  p.scale_log2 = static_cast<float>(static_cast<double>(c.scale) * 1.4426950408889634074);
  p.timeout_ns = wait_timeout_ns();
  // Persistent: as many 2-CTA clusters as can be resident at once, but never
  // more than tiles could exist.
  const long long max_tiles = static_cast<long long>(capacity) * c.num_heads * c.nsplit;
  const long long resident = g_dev[dev].dense_clusters.load(std::memory_order_relaxed);
  const long long clusters = max_tiles < resident ? max_tiles : resident;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t le;
  if (c.qk_dim == 192) {
    cfg.dynamicSmemBytes = Geo<192>::kSmemBytes;
    le = cudaLaunchKernelEx(&cfg, dense_fwd_kernel<192>, tq, tk, tv, tkc, tvc, p);
  } else if (c.qk_dim == 256) {
    cfg.dynamicSmemBytes = Geo<256>::kSmemBytes;
    le = cudaLaunchKernelEx(&cfg, dense_fwd_kernel<256>, tq, tk, tv, tkc, tvc, p);
  } else {
    cfg.dynamicSmemBytes = Geo<128>::kSmemBytes;
    le = cudaLaunchKernelEx(&cfg, dense_fwd_kernel<128>, tq, tk, tv, tkc, tvc, p);
  }
  if (le != cudaSuccess) {
    cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  if ((st = launch_status()) != MLA_OK || c.nsplit == 1) return st;
  // split-KV: combine the partials of every (token, head) row
  namespace mg = mla::merge;
  const long long rows = static_cast<long long>(c.total_q) * c.num_heads;
  const long long warps_per_block = mg::kCombineThreads / 32;
  const long long want = (rows + warps_per_block - 1) / warps_per_block;
  const long long cap = static_cast<long long>(g_dev[dev].sms.load(std::memory_order_relaxed)) * 8;
  mg::combine_splits_kernel<<<static_cast<unsigned>(want < cap ? want : cap), mg::kCombineThreads, 0,
                              s>>>(reinterpret_cast<const float4*>(p.o_part), p.lse_part, c.nsplit,
                                   c.total_q, c.num_heads, static_cast<uint2*>(c.out), c.lse);
  return launch_status();
}

// The call over packed q [T, H, 192], k [Tk, H, 192], v [Tk, H, 128].
DenseCall packed_call(const void* q, const void* k, const void* v, int num_heads) {
  using mla::dense::kDqk;
  using mla::dense::kDv;
  DenseCall c;
  const int64_t H = num_heads;
  c.q = q;
  c.q_rs = H * kDqk;
  c.q_hs = kDqk;
  c.k = k;
  c.k_rs = H * kDqk;
  c.k_hs = kDqk;
  c.v = v;
  c.v_rs = H * kDv;
  c.v_hs = kDv;
  return c;
}

}  // namespace

extern "C" {

int mla_prefill_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_k, int max_seqlen_q, int max_seqlen_k,
                    float softmax_scale, int causal, void* out, float* lse, mla_stream_t stream,
                    int batch, int num_heads, int total_q, int total_k, void* workspace,
                    size_t workspace_bytes) {
  using mla::dense::kDqk;
  using mla::dense::kDv;
  const int64_t H = num_heads;
  return mla_prefill_fwd_strided(q, H * kDqk, kDqk, k, H * kDqk, kDqk, v, H * kDv, kDv,
                                 cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                                 softmax_scale, causal, out, lse, stream, batch, num_heads,
                                 total_q, total_k, workspace, workspace_bytes);
}

int mla_prefill_fwd_strided(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                            const void* k, int64_t k_row_stride, int64_t k_head_stride,
                            const void* v, int64_t v_row_stride, int64_t v_head_stride,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                            void* out, float* lse, mla_stream_t stream, int batch, int num_heads,
                            int total_q, int total_k, void* workspace, size_t workspace_bytes) {
  DenseCall c;
  c.q = q;
  c.q_rs = q_row_stride;
  c.q_hs = q_head_stride;
  c.k = k;
  c.k_rs = k_row_stride;
  c.k_hs = k_head_stride;
  c.v = v;
  c.v_rs = v_row_stride;
  c.v_hs = v_head_stride;
  c.cu_q = cu_seqlens_q;
  c.cu_k = cu_seqlens_k;
  c.max_q = max_seqlen_q;
  c.max_k = max_seqlen_k;
  c.scale = softmax_scale;
  c.causal = causal;
  c.out = out;
  c.lse = lse;
  c.stream = stream;
  c.batch = batch;
  c.num_heads = num_heads;
  c.total_q = total_q;
  c.total_k = total_k;
  c.workspace = workspace;
  c.workspace_bytes = workspace_bytes;
  return dense_call(c);
}

int mla_prefill_fwd_context(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            const void* k_ctx, const void* v_ctx, const int32_t* cu_seqlens_ctx,
                            int max_seqlen_q, int max_seqlen_k, int max_seqlen_ctx,
                            float softmax_scale, int causal, void* out, float* lse,
                            mla_stream_t stream, int batch, int num_heads, int total_q,
                            int total_k, int total_ctx, void* workspace, size_t workspace_bytes) {
  if (k_ctx == nullptr || v_ctx == nullptr || cu_seqlens_ctx == nullptr)
    return MLA_ERR_INVALID_ARG;
  DenseCall c = packed_call(q, k, v, num_heads);
  c.cu_q = cu_seqlens_q;
  c.cu_k = cu_seqlens_k;
  c.k_ctx = k_ctx;
  c.v_ctx = v_ctx;
  c.cu_ctx = cu_seqlens_ctx;
  c.max_ctx = max_seqlen_ctx;
  c.total_ctx = total_ctx;
  c.max_q = max_seqlen_q;
  c.max_k = max_seqlen_k;
  c.scale = softmax_scale;
  c.causal = causal;
  c.out = out;
  c.lse = lse;
  c.stream = stream;
  c.batch = batch;
  c.num_heads = num_heads;
  c.total_q = total_q;
  c.total_k = total_k;
  c.workspace = workspace;
  c.workspace_bytes = workspace_bytes;
  return dense_call(c);
}

size_t mla_prefill_splitkv_workspace_size(int batch, int total_q, int num_heads, int num_splits) {
  const size_t base = mla_prefill_workspace_size(batch, total_q);
  if (base == 0 || num_heads < 1 || num_splits < 1 || num_splits > MLA_MAX_SPLITS) return 0;
  if (num_splits == 1) return base;
  const size_t rows = static_cast<size_t>(total_q) * static_cast<size_t>(num_heads);
  return splitkv_parts_offset(base) +
         static_cast<size_t>(num_splits) * rows * (mla::dense::kDv + 1) * sizeof(float);
}

int mla_prefill_num_splits(int batch, int total_q, int num_heads, int max_seqlen_q,
                           int max_seqlen_k) {
  if (batch < 1 || total_q < 0 || num_heads < 1 || max_seqlen_q < 0 || max_seqlen_k < 0) return 1;
  using mla::dense::kBlockKeys;
  using mla::dense::kTileRows;
  int dev = 0;
  int clusters = 74;  // the B200's 148 SMs as CTA pairs, if no device is current
  if (prepare_device(&dev) == MLA_OK)
    clusters = g_dev[dev].dense_clusters.load(std::memory_order_relaxed);
  // tiles the call has at most: (sequence, 512-row block) entries x heads
  const long long per_seq = (static_cast<long long>(max_seqlen_q) + kTileRows - 1) / kTileRows;
  const long long by_total = (static_cast<long long>(total_q) + kTileRows - 1) / kTileRows + batch;
  const long long entries = per_seq * batch < by_total ? per_seq * batch : by_total;
  const long long tiles = entries * num_heads;
  if (tiles <= 0 || tiles >= clusters) return 1;
  const long long blocks = (static_cast<long long>(max_seqlen_k) + kBlockKeys - 1) / kBlockKeys;
  long long n_max = blocks / 2;                               // at least two KV blocks a split
  if (n_max > MLA_MAX_SPLITS) n_max = MLA_MAX_SPLITS;
  // The fewest splits that minimise the critical path: waves of split tiles
  // over the clusters times the blocks of one split, plus about two blocks'
  // worth of per-tile overhead (Q load, partial store).
  long long best_n = 1, best_cost = -1;
  for (long long n = 1; n <= n_max; ++n) {
    const long long waves = (tiles * n + clusters - 1) / clusters;
    const long long cost = waves * ((blocks + n - 1) / n + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_n = n;
    }
  }
  return static_cast<int>(best_n);
}

int mla_prefill_fwd_splitkv(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                            int num_splits, void* out, float* lse, mla_stream_t stream, int batch,
                            int num_heads, int total_q, int total_k, void* workspace,
                            size_t workspace_bytes) {
  DenseCall c = packed_call(q, k, v, num_heads);
  c.cu_q = cu_seqlens_q;
  c.cu_k = cu_seqlens_k;
  c.nsplit = num_splits;
  c.max_q = max_seqlen_q;
  c.max_k = max_seqlen_k;
  c.scale = softmax_scale;
  c.causal = causal;
  c.out = out;
  c.lse = lse;
  c.stream = stream;
  c.batch = batch;
  c.num_heads = num_heads;
  c.total_q = total_q;
  c.total_k = total_k;
  c.workspace = workspace;
  c.workspace_bytes = workspace_bytes;
  return dense_call(c);
}

int mla_prefill_fwd_dims(const void* q, const void* k, const void* v,
                         const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                         int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                         void* out, float* lse, mla_stream_t stream, int batch, int num_heads,
                         int total_q, int total_k, int qk_dim, int v_dim, void* workspace,
                         size_t workspace_bytes) {
  using mla::dense::kDv;
  if ((qk_dim != 128 && qk_dim != 192 && qk_dim != 256) || (v_dim != 128 && v_dim != 256) ||
      num_heads < 1)
    return MLA_ERR_INVALID_ARG;
  // One pass per 128 value dims: pass j reads v[..., 128 j : 128 j + 128] and
  // writes out[..., 128 j : 128 j + 128] (strided views); the scores, and so
  // the LSE, are the same in every pass, which writes it only in the first.
  const int passes = v_dim / kDv;
  const int64_t H = num_heads;
  for (int j = 0; j < passes; ++j) {
    DenseCall c;
    c.q = q;
    c.q_rs = H * qk_dim;
    c.q_hs = qk_dim;
    c.k = k;
    c.k_rs = H * qk_dim;
    c.k_hs = qk_dim;
    c.v = v == nullptr ? nullptr : static_cast<const char*>(v) + static_cast<size_t>(j) * kDv * 2;
    c.v_rs = H * v_dim;
    c.v_hs = v_dim;
    c.qk_dim = qk_dim;
    c.out = out == nullptr ? nullptr : static_cast<char*>(out) + static_cast<size_t>(j) * kDv * 2;
    c.out_rs = H * v_dim;
    c.out_hs = v_dim;
    c.cu_q = cu_seqlens_q;
    c.cu_k = cu_seqlens_k;
    c.max_q = max_seqlen_q;
    c.max_k = max_seqlen_k;
    c.scale = softmax_scale;
    c.causal = causal;
    c.lse = j == 0 ? lse : nullptr;
    c.stream = stream;
    c.batch = batch;
    c.num_heads = num_heads;
    c.total_q = total_q;
    c.total_k = total_k;
    c.workspace = workspace;
    c.workspace_bytes = workspace_bytes;
    const int st = dense_call(c);
    if (st != MLA_OK) return st;
  }
  return MLA_OK;
}

int mla_prefill_fwd_ex(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                       const int32_t* cu_seqlens_k, int max_seqlen_q, int max_seqlen_k,
                       float softmax_scale, int causal, const float* sinks,
                       const float* output_scale, void* out, float* lse, mla_stream_t stream,
                       int batch, int num_heads, int total_q, int total_k, void* workspace,
                       size_t workspace_bytes) {
  DenseCall c = packed_call(q, k, v, num_heads);
  c.cu_q = cu_seqlens_q;
  c.cu_k = cu_seqlens_k;
  c.sinks = sinks;
  c.out_scale = output_scale;
  c.max_q = max_seqlen_q;
  c.max_k = max_seqlen_k;
  c.scale = softmax_scale;
  c.causal = causal;
  c.out = out;
  c.lse = lse;
  c.stream = stream;
  c.batch = batch;
  c.num_heads = num_heads;
  c.total_q = total_q;
  c.total_k = total_k;
  c.workspace = workspace;
  c.workspace_bytes = workspace_bytes;
  return dense_call(c);
}

int mla_prefill_fwd_noalloc(const void* q, const void* k, const void* v,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            int max_seqlen_q, int max_seqlen_k, float softmax_scale, int causal,
                            void* out, float* lse, mla_stream_t stream, int batch, int num_heads,
                            int total_q, int total_k) {
  const size_t need = mla_prefill_workspace_size(batch, total_q);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (need > MLA_NOALLOC_SCRATCH_BYTES) return MLA_ERR_SCRATCH_TOO_SMALL;
  int dev = 0;
  int st = prepare_device(&dev);
  if (st != MLA_OK) return st;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(dev, &scratch)) != MLA_OK) return st;
  return mla_prefill_fwd(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                         softmax_scale, causal, out, lse, stream, batch, num_heads, total_q,
                         total_k, scratch, MLA_NOALLOC_SCRATCH_BYTES);
}

int mla_attn_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                   void* out, float* lse_out, int num_tokens, int num_heads, int head_dim,
                   mla_stream_t stream) {
  if (o_a == nullptr || o_b == nullptr || lse_a == nullptr || lse_b == nullptr || out == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(o_a, 16) || !aligned(o_b, 16) || !aligned(out, 16) || !aligned(lse_a, 4) ||
      !aligned(lse_b, 4) || (lse_out && !aligned(lse_out, 4)))
    return MLA_ERR_INVALID_ARG;
  if (lse_out != nullptr && (lse_out == lse_a || lse_out == lse_b)) return MLA_ERR_INVALID_ARG;
  if (num_tokens < 0 || num_heads < 1 || head_dim < 8 || head_dim % 8 != 0)
    return MLA_ERR_INVALID_ARG;
  int dev = 0;
  int st = prepare_device(&dev);
  if (st != MLA_OK) return st;
  if (num_tokens == 0) return MLA_OK;
  const long long rows = static_cast<long long>(num_tokens) * num_heads;
  const int vpr = head_dim / 8;
  const long long vecs = rows * vpr;
  const int sms = g_dev[dev].sms.load(std::memory_order_relaxed);
  const long long want = (vecs + mla::merge::kThreads - 1) / mla::merge::kThreads;
  const long long cap = static_cast<long long>(sms) * 8;  // 8 resident CTAs of 256 per SM
  const int blocks = static_cast<int>(want < cap ? want : cap);
  mla::merge::merge_kernel<<<blocks, mla::merge::kThreads, 0,
                             reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(o_a), lse_a, static_cast<const uint4*>(o_b), lse_b,
      static_cast<uint4*>(out), lse_out, rows, num_heads, num_tokens, vpr);
  return launch_status();
}

int mla_sparse_prefill_fwd(const void* q, const void* kv_latent, const int32_t* indices, int topk,
                           float softmax_scale, void* out, float* lse, mla_stream_t stream,
                           int num_tokens, int num_heads, int num_kv_rows) {
  if (q == nullptr || kv_latent == nullptr || indices == nullptr || out == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv_latent, 16) || !aligned(out, 16) || !aligned(indices, 4) ||
      (lse && !aligned(lse, 4)))
    return MLA_ERR_INVALID_ARG;
  if (topk < 1 || num_tokens < 0 || num_heads < 1 || num_heads > 128 || num_kv_rows < 1)
    return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.0f)) return MLA_ERR_INVALID_ARG;
  // grid = 2 CTAs per token (an int); TMA row coordinates are int32
  if (2 * static_cast<int64_t>(num_tokens) > INT32_MAX ||
      static_cast<int64_t>(num_tokens) * num_heads > INT32_MAX)
    return MLA_ERR_INVALID_ARG;
  int dev = 0;
  int st = prepare_device(&dev);
  if (st != MLA_OK) return st;
  if (num_tokens == 0) return MLA_OK;
  namespace sp = mla::sparse;
  CUtensorMap tm_q;
  if ((st = encode_rows(&tm_q, q, sp::kDl, static_cast<uint64_t>(num_tokens) * num_heads, sp::kM)) !=
      MLA_OK)
    return st;
  sp::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kv = static_cast<const __nv_bfloat16*>(kv_latent);
  p.indices = indices;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.num_tokens = num_tokens;
  p.num_heads = num_heads;
  p.num_rows = num_kv_rows;
  p.topk = topk;
  p.scale_log2 = static_cast<float>(static_cast<double>(softmax_scale) * 1.4426950408889634074);
  p.wide_out = aligned(out, 32) ? 1 : 0;  // rows of 1024 bytes, halves of 512
  p.timeout_ns = wait_timeout_ns();
  sp::sparse_fwd_kernel<<<2 * num_tokens, sp::kThreads, sp::kSmemBytes,
                          reinterpret_cast<cudaStream_t>(stream)>>>(tm_q, p);
  return launch_status();
}

int mla_device_status(unsigned int* status, int reset) {
  if (status == nullptr) return MLA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpyFromSymbol(status, mla::g_mla_status, sizeof(unsigned int)) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (reset) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(mla::g_mla_status, &zero, sizeof(zero)) != cudaSuccess)
      return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

int mla_debug_wait_timeout(int timeout_us, mla_stream_t stream) {
  if (timeout_us < 1 || timeout_us > 10000000) return MLA_ERR_INVALID_ARG;
  int dev = 0;
  int st = prepare_device(&dev);
  if (st != MLA_OK) return st;
  wait_timeout_probe<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_us) * 1000ull);
  return launch_status();
}

}  // extern "C"
