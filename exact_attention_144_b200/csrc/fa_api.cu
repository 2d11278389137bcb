// fa_api.cu -- the C ABI: argument validation, device checks, TMA tensor-map
// encoding and the device status word.  No torch types cross this boundary.
#include <math.h>
#include <atomic>
#include <mutex>

#include "fa_common.cuh"
#include "fa_host.h"

namespace fa {

__device__ unsigned long long g_status = 0;

static std::atomic<unsigned long long> g_launches{0};
static std::atomic<int> g_last_cuda_error{0};

int launch_status(cudaError_t e) {
  if (e == cudaSuccess) return FA_OK;
  g_last_cuda_error.store((int)e);
  return FA_ERR_LAUNCH;
}

int check_launch_regs(const void* kernel) {
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, kernel);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return launch_status(e);
  }
  return attr.numRegs >= kLaunchRegs ? FA_OK : launch_status(cudaErrorInvalidConfiguration);
}
static std::mutex g_event_mu;
static cudaEvent_t g_events[4] = {nullptr, nullptr, nullptr, nullptr};

void note_launches(unsigned n) { g_launches.fetch_add(n); }

void take_kernel_events(bool bwd, cudaEvent_t* start, cudaEvent_t* stop) {
  std::lock_guard<std::mutex> lock(g_event_mu);
  const int i = bwd ? 2 : 0;
  *start = g_events[i];
  *stop = g_events[i + 1];
  g_events[i] = g_events[i + 1] = nullptr;
}

static void arm_kernel_events(cudaEvent_t fs, cudaEvent_t fe, cudaEvent_t bs, cudaEvent_t be) {
  std::lock_guard<std::mutex> lock(g_event_mu);
  g_events[0] = fs;
  g_events[1] = fe;
  g_events[2] = bs;
  g_events[3] = be;
}

// ------------------------------------------------------- context identity
// Device addresses of __device__ variables and memory pools belong to a CUDA
// context, not to a device number: after cudaDeviceReset, or with another
// context current, the old values are stale.  Cached values are therefore
// keyed by the unique ID of the context current on the calling thread
// (cuCtxGetId, reached through the runtime's driver entry points).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

static void* driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult qres;
  if (cudaGetDriverEntryPointByVersion(name, &ptr, 12000, cudaEnableDefault, &qres) !=
          cudaSuccess ||
      qres != cudaDriverEntryPointSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return ptr;
}

bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_current = reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
    get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
  });
  CUcontext ctx = nullptr;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr)
    return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Small table of (context ID, key) -> value, replaced round-robin when full.
struct ContextCache {
  struct Entry {
    unsigned long long ctx;
    const void* key;
    void* value;
  };
  std::mutex mu;
  Entry e[64] = {};
  int n = 0, next = 0;
  bool find(unsigned long long ctx, const void* key, void** value) {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
      if (e[i].ctx == ctx && e[i].key == key) {
        *value = e[i].value;
        return true;
      }
    return false;
  }
  void insert(unsigned long long ctx, const void* key, void* value) {
    std::lock_guard<std::mutex> lock(mu);
    const int i = n < 64 ? n++ : (next++ % 64);
    e[i] = {ctx, key, value};
  }
};

int symbol_address(const void* symbol, void** out) {
  static ContextCache cache;
  unsigned long long ctx = 0;
  bool have = current_context_id(&ctx);
  if (have && cache.find(ctx, symbol, out)) return FA_OK;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, symbol) != cudaSuccess || ptr == nullptr) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  if (!have) have = current_context_id(&ctx);  // the lookup made a context current
  if (have) cache.insert(ctx, symbol, ptr);
  *out = ptr;
  return FA_OK;
}

unsigned long long* device_status_ptr() {
  void* ptr = nullptr;
  return symbol_address(&g_status, &ptr) == FA_OK ? static_cast<unsigned long long*>(ptr)
                                                  : nullptr;
}

// ------------------------------------------------------------ scratch pool
static std::atomic<unsigned long long> g_scratch_allocs{0};

// The library's memory pool for device dev in the current context.
static cudaMemPool_t scratch_pool(int dev) {
  static ContextCache cache;
  static std::mutex create_mu;
  const void* key = reinterpret_cast<const void*>((uintptr_t)dev + 1);
  unsigned long long ctx = 0;
  bool have = current_context_id(&ctx);
  void* found = nullptr;
  if (have && cache.find(ctx, key, &found)) return static_cast<cudaMemPool_t>(found);
  std::lock_guard<std::mutex> lock(create_mu);
  if (have && cache.find(ctx, key, &found)) return static_cast<cudaMemPool_t>(found);
  cudaMemPoolProps props{};
  props.allocType = cudaMemAllocationTypePinned;
  props.handleTypes = cudaMemHandleTypeNone;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = dev;
  cudaMemPool_t pool = nullptr;
  if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  unsigned long long keep = kScratchRetainBytes;
  if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess)
    cudaGetLastError();  // still usable, only without retention
  if (!have) have = current_context_id(&ctx);
  if (have) cache.insert(ctx, key, pool);
  return pool;
}

unsigned long long scratch_allocs() { return g_scratch_allocs.load(); }

int scratch_alloc(void** ptr, size_t bytes, cudaStream_t stream) {
  g_scratch_allocs.fetch_add(1);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_NOMEM;
  }
  if (dev < 0) return FA_ERR_NOMEM;
  cudaMemPool_t pool = scratch_pool(dev);
  if (pool == nullptr || cudaMallocFromPoolAsync(ptr, bytes, pool, stream) != cudaSuccess) {
    cudaGetLastError();
    *ptr = nullptr;
    return FA_ERR_NOMEM;
  }
  return FA_OK;
}

void scratch_free(void* ptr, cudaStream_t stream) {
  if (ptr != nullptr && cudaFreeAsync(ptr, stream) != cudaSuccess) cudaGetLastError();
}

// ------------------------------------------------------------ device info
int current_device(DeviceInfo* info) {
  static std::mutex mu;
  static int cached_sm[64] = {0};
  static int cached_smem[64] = {0};
  static int cached_ok[64] = {0};  // 0 unknown, 1 sm_100, -1 other
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  if (dev < 0 || dev >= 64) return FA_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (cached_ok[dev] == 0) {
    int major = 0, minor = 0, sms = 0, smem = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_LAUNCH;
    }
    cached_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    cached_sm[dev] = sms;
    cached_smem[dev] = smem;
  }
  if (cached_ok[dev] != 1) return FA_ERR_DEVICE;
  info->device = dev;
  info->sm_count = cached_sm[dev];
  info->max_smem_optin = cached_smem[dev];
  return FA_OK;
}

// ------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &qres) == cudaSuccess &&
        qres == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    else
      cudaGetLastError();
  });
  return fn;
}

int make_tmap_bnhd(CUtensorMap* map, const void* base, int fmt, int B, int N, int H, int d,
                   int box_rows, long long tok_stride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FA_ERR_LAUNCH;
  const cuuint64_t eb = fmt == 2 ? 1 : 2;  // bytes an element
  // dims innermost first: element within head, head, token, batch
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * eb, (cuuint64_t)tok_stride * eb,
                                 (cuuint64_t)N * tok_stride * eb};
  const cuuint32_t box[4] = {(cuuint32_t)(128 / eb), 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = fmt == 2   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                 : fmt == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUresult r = fn(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_LAUNCH;
}

int make_tmap_f32_rows(CUtensorMap* map, const void* base, size_t rows, int cols, int box_cols,
                       int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FA_ERR_LAUNCH;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_LAUNCH;
}

// ------------------------------------------------------------ validation
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape, head-size and scale checks shared by every entry point (the 8-bit
// forward then narrows d to 128).
static int check_common(int B, int H, int N, int d, float scale) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_SHAPE;
  if (!(d == 64 || d == 96 || d == 128 || d == 256)) return FA_ERR_HEADDIM;
  if ((long long)B * N * H * d >= (1ll << 31)) return FA_ERR_SHAPE;
  if (!isfinite(scale)) return FA_ERR_SCALE;
  return FA_OK;
}

static int check_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs)
    if (p == nullptr) return FA_ERR_NULL;
  for (const void* p : ptrs)
    if (!aligned16(p)) return FA_ERR_ALIGN;
  return FA_OK;
}

template <class T>
static int fwd_entry(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int N, int d, float scale, unsigned flags, cudaStream_t stream) {
  int rc = check_ptrs({q, k, v, o, lse});
  if (rc == FA_OK) rc = check_common(B, H, N, d, scale);
  if (rc == FA_OK && (flags & ~kKnownFlags) != 0) rc = FA_ERR_FLAGS;
  if (rc == FA_OK)
    rc = fwd_launch<T>(q, k, v, o, lse, B, H, N, d, scale, flags, (long long)H * d, stream);
  return rc;
}

template <class T>
static int bwd_entry(const void* q, const void* k, const void* v, const void* o, const void* dout,
                     const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                     float scale, unsigned flags, cudaStream_t stream) {
  int rc = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv});
  if (rc == FA_OK) rc = check_common(B, H, N, d, scale);
  if (rc == FA_OK && (flags & ~kKnownFlags) != 0) rc = FA_ERR_FLAGS;
  if (rc == FA_OK)
    rc = bwd_launch<T>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, flags,
                       (long long)H * d, (long long)H * d, stream);
  return rc;
}

// Packed Q, K, V: qkv is [B, N, 3, H, d]; Q, K, V are its slices 0, 1, 2
// (token stride 3*H*d), and dqkv the same for the gradients.
template <class T>
static int fwd_packed_entry(const void* qkv, void* o, float* lse, int B, int H, int N, int d,
                            float scale, unsigned flags, cudaStream_t stream) {
  int rc = check_ptrs({qkv, o, lse});
  if (rc == FA_OK) rc = check_common(B, H, N, d, scale);
  if (rc == FA_OK && (long long)B * N * 3 * H * d >= (1ll << 31)) rc = FA_ERR_SHAPE;
  if (rc == FA_OK && (flags & ~kKnownFlags) != 0) rc = FA_ERR_FLAGS;
  if (rc != FA_OK) return rc;
  const T* base = static_cast<const T*>(qkv);
  const long long hd = (long long)H * d;
  return fwd_launch<T>(base, base + hd, base + 2 * hd, o, lse, B, H, N, d, scale, flags, 3 * hd,
                       stream);
}

template <class T>
static int bwd_packed_entry(const void* qkv, const void* o, const void* dout, const float* lse,
                            void* dqkv, int B, int H, int N, int d, float scale, unsigned flags,
                            cudaStream_t stream) {
  int rc = check_ptrs({qkv, o, dout, lse, dqkv});
  if (rc == FA_OK) rc = check_common(B, H, N, d, scale);
  if (rc == FA_OK && (long long)B * N * 3 * H * d >= (1ll << 31)) rc = FA_ERR_SHAPE;
  if (rc == FA_OK && (flags & ~kKnownFlags) != 0) rc = FA_ERR_FLAGS;
  if (rc != FA_OK) return rc;
  const T* base = static_cast<const T*>(qkv);
  T* g = static_cast<T*>(dqkv);
  const long long hd = (long long)H * d;
  return bwd_launch<T>(base, base + hd, base + 2 * hd, o, dout, lse, g, g + hd, g + 2 * hd, B, H,
                       N, d, scale, flags, 3 * hd, 3 * hd, stream);
}

// E4M3 Q, K, V with per-tensor descale factors: the problem is attention on
// (descale_q Q, descale_k K, descale_v V); O is bf16.
static int fwd_fp8_entry(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int N, int d, float scale, float descale_q, float descale_k,
                         float descale_v, unsigned flags, cudaStream_t stream) {
  int rc = check_ptrs({q, k, v, o, lse});
  if (rc == FA_OK) rc = check_common(B, H, N, d, scale);
  if (rc == FA_OK && d != 128) rc = FA_ERR_HEADDIM;
  const float s_eff = scale * descale_q * descale_k;
  if (rc == FA_OK && !(isfinite(descale_q) && isfinite(descale_k) && isfinite(descale_v) &&
                       isfinite(s_eff)))
    rc = FA_ERR_SCALE;
  if (rc == FA_OK && (flags & ~kKnownFlags) != 0) rc = FA_ERR_FLAGS;
  if (rc == FA_OK)
    rc = fwd_launch<__nv_fp8_e4m3>(q, k, v, o, lse, B, H, N, d, s_eff, flags, (long long)H * d,
                                   stream, nullptr, 0, descale_v);
  return rc;
}

// Variable-length batch: B sequences packed along one token axis of `total`
// tokens ([total, H, d] tensors, lse [H, total]); cu_seqlens (device, B + 1
// entries) holds each sequence's first token, max_seqlen bounds their lengths.
static int check_varlen(const int* cu, int B, int total, int max_seqlen, int H, int d,
                        float scale) {
  if (cu == nullptr) return FA_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(cu) & 3u) != 0) return FA_ERR_ALIGN;
  if (total < 1 || max_seqlen < 1) return FA_ERR_SHAPE;
  int rc = check_common(B, H, max_seqlen, d, scale);
  if (rc == FA_OK && (long long)total * H * d >= (1ll << 31)) rc = FA_ERR_SHAPE;
  return rc;
}

template <class T>
static int fwd_varlen_entry(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu, int B, int total, int max_seqlen, int H, int d,
                            float scale, unsigned flags, cudaStream_t stream) {
  int rc = check_ptrs({q, k, v, o, lse});
  if (rc == FA_OK) rc = check_varlen(cu, B, total, max_seqlen, H, d, scale);
  if (rc == FA_OK && (flags & ~kKnownFlags) != 0) rc = FA_ERR_FLAGS;
  if (rc != FA_OK) return rc;
  return fwd_launch<T>(q, k, v, o, lse, B, H, max_seqlen, d, scale, flags, (long long)H * d,
                       stream, cu, total);
}

template <class T>
static int bwd_varlen_entry(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv,
                            const int* cu, int B, int total, int max_seqlen, int H, int d,
                            float scale, unsigned flags, cudaStream_t stream) {
  int rc = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv});
  if (rc == FA_OK) rc = check_varlen(cu, B, total, max_seqlen, H, d, scale);
  if (rc == FA_OK && (flags & ~kKnownFlags) != 0) rc = FA_ERR_FLAGS;
  if (rc != FA_OK) return rc;
  return bwd_launch<T>(q, k, v, o, dout, lse, dq, dk, dv, B, H, max_seqlen, d, scale, flags,
                       (long long)H * d, (long long)H * d, stream, cu, total);
}

int check_bwd_args(const void* q, const void* k, const void* v, const void* o, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                   float scale) {
  int rc = check_ptrs({q, k, v, o, dout, lse, dq, dk, dv});
  if (rc == FA_OK) rc = check_common(B, H, N, d, scale);
  return rc;
}

// ---------------------------------------------------- bounded-wait test
__global__ void selftest_wait_kernel(unsigned long long limit_ns, unsigned long long* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    // expects two arrivals; only one ever comes, so the phase never completes
    mbar_init(smem_u32(&bar), 2);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive(smem_u32(&bar));
    const WaitCtl w{&abort_flag, limit_ns, status};
    mbar_wait(smem_u32(&bar), 0, w, 0x7F);
  }
  __syncthreads();
}

// y = 2^x by ex2_poly2 (the FMA-pipe exponential of the softmax), two per thread
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : x[i];
  float ya, yb;
  ex2_poly2(ya, yb, a, b);
  y[i] = ya;
  if (i + 1 < n) y[i + 1] = yb;
}

}  // namespace fa

// =================================================================== C ABI
// Only these entry points are visible outside the library.
#define FA_EXPORT __attribute__((visibility("default")))

extern "C" {

FA_EXPORT int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, float scale, cudaStream_t stream) {
  return fa::fwd_entry<__nv_bfloat16>(q, k, v, o, lse, B, H, N, d, scale, 0u, stream);
}

FA_EXPORT int fa_fwd_f16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int N, int d, float scale, cudaStream_t stream) {
  return fa::fwd_entry<__half>(q, k, v, o, lse, B, H, N, d, scale, 0u, stream);
}

FA_EXPORT int fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int N, int d, float scale, int dtype, unsigned flags,
                        cudaStream_t stream) {
  if (dtype == FA_BF16)
    return fa::fwd_entry<__nv_bfloat16>(q, k, v, o, lse, B, H, N, d, scale, flags, stream);
  if (dtype == FA_FP16)
    return fa::fwd_entry<__half>(q, k, v, o, lse, B, H, N, d, scale, flags, stream);
  return FA_ERR_DTYPE;
}

FA_EXPORT int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int N, int d, float scale, float descale_q, float descale_k,
                         float descale_v, unsigned flags, cudaStream_t stream) {
  return fa::fwd_fp8_entry(q, k, v, o, lse, B, H, N, d, scale, descale_q, descale_k, descale_v,
                           flags, stream);
}

FA_EXPORT int fa_fwd_qkvpacked(const void* qkv, void* o, float* lse, int B, int H, int N, int d,
                               float scale, int dtype, unsigned flags, cudaStream_t stream) {
  if (dtype == FA_BF16)
    return fa::fwd_packed_entry<__nv_bfloat16>(qkv, o, lse, B, H, N, d, scale, flags, stream);
  if (dtype == FA_FP16)
    return fa::fwd_packed_entry<__half>(qkv, o, lse, B, H, N, d, scale, flags, stream);
  return FA_ERR_DTYPE;
}

FA_EXPORT int fa_bwd_qkvpacked(const void* qkv, const void* o, const void* dout, const float* lse,
                               void* dqkv, int B, int H, int N, int d, float scale, int dtype,
                               unsigned flags, cudaStream_t stream) {
  if (dtype == FA_BF16)
    return fa::bwd_packed_entry<__nv_bfloat16>(qkv, o, dout, lse, dqkv, B, H, N, d, scale, flags,
                                               stream);
  if (dtype == FA_FP16)
    return fa::bwd_packed_entry<__half>(qkv, o, dout, lse, dqkv, B, H, N, d, scale, flags, stream);
  return FA_ERR_DTYPE;
}

FA_EXPORT int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu_seqlens, int B, int total, int max_seqlen, int H, int d,
                            float scale, int dtype, unsigned flags, cudaStream_t stream) {
  if (dtype == FA_BF16)
    return fa::fwd_varlen_entry<__nv_bfloat16>(q, k, v, o, lse, cu_seqlens, B, total, max_seqlen,
                                               H, d, scale, flags, stream);
  if (dtype == FA_FP16)
    return fa::fwd_varlen_entry<__half>(q, k, v, o, lse, cu_seqlens, B, total, max_seqlen, H, d,
                                        scale, flags, stream);
  return FA_ERR_DTYPE;
}

FA_EXPORT int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                            const void* dout, const float* lse, void* dq, void* dk, void* dv,
                            const int* cu_seqlens, int B, int total, int max_seqlen, int H, int d,
                            float scale, int dtype, unsigned flags, cudaStream_t stream) {
  if (dtype == FA_BF16)
    return fa::bwd_varlen_entry<__nv_bfloat16>(q, k, v, o, dout, lse, dq, dk, dv, cu_seqlens, B,
                                               total, max_seqlen, H, d, scale, flags, stream);
  if (dtype == FA_FP16)
    return fa::bwd_varlen_entry<__half>(q, k, v, o, dout, lse, dq, dk, dv, cu_seqlens, B, total,
                                        max_seqlen, H, d, scale, flags, stream);
  return FA_ERR_DTYPE;
}

FA_EXPORT int fa_varlen_bounds(const int* cu_seqlens_host, int b, int max_seqlen, int total,
                               int* tok0, int* len) {
  if (cu_seqlens_host == nullptr || tok0 == nullptr || len == nullptr) return FA_ERR_NULL;
  if (b < 0 || max_seqlen < 1 || total < 1) return FA_ERR_SHAPE;
  int tb = 0;
  fa::seq_bounds(cu_seqlens_host, b, max_seqlen, total, tb, *tok0, *len);
  return FA_OK;
}

FA_EXPORT int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
           const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale,
           cudaStream_t stream) {
  return fa::bwd_entry<__nv_bfloat16>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, 0u,
                                      stream);
}

FA_EXPORT int fa_bwd_f16(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
               float scale, cudaStream_t stream) {
  return fa::bwd_entry<__half>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, 0u, stream);
}

FA_EXPORT int fa_bwd_ex(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                        int H, int N, int d, float scale, int dtype, unsigned flags,
                        cudaStream_t stream) {
  if (dtype == FA_BF16)
    return fa::bwd_entry<__nv_bfloat16>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale,
                                        flags, stream);
  if (dtype == FA_FP16)
    return fa::bwd_entry<__half>(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, flags,
                                 stream);
  return FA_ERR_DTYPE;
}

FA_EXPORT int fa_fwd_plan_ex(int B, int H, int N, int d, unsigned flags, int sm_count,
                             fa_fwd_plan_t* plan) {
  if (plan == nullptr) return FA_ERR_NULL;
  if ((flags & ~fa::kKnownFlags) != 0) return FA_ERR_FLAGS;
  fa::FwdSchedule s;
  const int rc = fa::plan_fwd(B, H, N, d, flags, sm_count, &s);
  if (rc != FA_OK) return rc;
  plan->kernel = s.pair;
  plan->unit_rows = s.unit_rows;
  plan->kv_tile_rows = s.bn;
  plan->n_units = s.n_units;
  plan->n_kv_tiles = s.n_kvt;
  plan->n_split = s.n_split;
  plan->grid = s.grid;
  plan->balanced = s.n_iter > 0 ? 1 : 0;
  plan->scratch_bytes = (long long)fa::fwd_scratch_bytes(s);
  return FA_OK;
}

FA_EXPORT int fa_fwd_plan(int B, int H, int N, int d, int sm_count, fa_fwd_plan_t* plan) {
  return fa_fwd_plan_ex(B, H, N, d, 0u, sm_count, plan);
}

FA_EXPORT int fa_bwd_plan(int B, int H, int N, int d, unsigned flags, int sm_count,
                          int* n_split, int* grid_blocks) {
  if (n_split == nullptr || grid_blocks == nullptr) return FA_ERR_NULL;
  if ((flags & ~fa::kKnownFlags) != 0) return FA_ERR_FLAGS;
  return fa::plan_bwd(B, H, N, d, flags, sm_count, n_split, grid_blocks);
}

FA_EXPORT int fa_fwd_plan_pieces_ex(int B, int H, int N, int d, unsigned flags, int sm_count,
                                    int block, int* pieces, int max_pieces) {
  if (pieces == nullptr && max_pieces > 0) return FA_ERR_NULL;
  if ((flags & ~fa::kKnownFlags) != 0) return FA_ERR_FLAGS;
  fa::FwdSchedule s;
  const int rc = fa::plan_fwd(B, H, N, d, flags, sm_count, &s);
  if (rc != FA_OK) return rc;
  if (block < 0 || block >= s.grid) return FA_ERR_SHAPE;
  return fa::fwd_block_pieces(s, block, pieces, max_pieces < 0 ? 0 : max_pieces);
}

FA_EXPORT int fa_fwd_plan_pieces(int B, int H, int N, int d, int sm_count, int block,
                                 int* pieces, int max_pieces) {
  return fa_fwd_plan_pieces_ex(B, H, N, d, 0u, sm_count, block, pieces, max_pieces);
}

FA_EXPORT const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_NULL: return "a required pointer is NULL";
    case FA_ERR_SHAPE: return "B, H or N below 1, or a tensor of 2^31 or more elements";
    case FA_ERR_HEADDIM: return "head dimension not supported by this entry point";
    case FA_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case FA_ERR_LAUNCH: return "the CUDA runtime rejected a launch or call";
    case FA_ERR_NOMEM: return "scratch allocation failed";
    case FA_ERR_DEVICE: return "current device is not compute capability 10.0 (B200)";
    case FA_ERR_SCALE: return "scale is NaN or infinite";
    case FA_ERR_SCRATCH: return "problem needs more scratch than the fixed no-alloc buffer (64 MiB) holds";
    case FA_ERR_FLAGS: return "unknown flag bits";
    case FA_ERR_DTYPE: return "unknown element type";
    default: return "unknown status";
  }
}

FA_EXPORT int fa_get_device_status(unsigned long long* status_out, int clear) {
  if (status_out == nullptr) return FA_ERR_NULL;
  unsigned long long v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_status, sizeof(v)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  *status_out = v;
  if (clear) {
    const unsigned long long zero = 0;
    if (cudaMemcpyToSymbol(fa::g_status, &zero, sizeof(zero)) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_LAUNCH;
    }
  }
  return FA_OK;
}

FA_EXPORT int fa_selftest_bounded_wait(unsigned int limit_us, unsigned long long* status_out) {
  if (status_out == nullptr) return FA_ERR_NULL;
  if (limit_us < 1 || limit_us > 10000000u) return FA_ERR_SHAPE;
  fa::DeviceInfo dev;
  int rc = fa::current_device(&dev);
  if (rc != FA_OK) return rc;
  unsigned long long prev = 0;
  if ((rc = fa_get_device_status(&prev, 1)) != FA_OK) return rc;
  fa::selftest_wait_kernel<<<1, 32>>>((unsigned long long)limit_us * 1000ull,
                                      fa::device_status_ptr());
  fa::note_launches(1);
  if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return fa_get_device_status(status_out, 1);
}

FA_EXPORT int fa_selftest_exp2(const float* x, float* y, int n, cudaStream_t stream) {
  if (x == nullptr || y == nullptr) return FA_ERR_NULL;
  if (n < 1) return FA_ERR_SHAPE;
  fa::DeviceInfo dev;
  int rc = fa::current_device(&dev);
  if (rc != FA_OK) return rc;
  const int pairs = (n + 1) / 2;
  fa::selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y, n);
  fa::note_launches(1);
  return fa::launch_status(cudaGetLastError());
}

FA_EXPORT int fa_set_kernel_events(cudaEvent_t fwd_start, cudaEvent_t fwd_stop,
                                   cudaEvent_t bwd_start, cudaEvent_t bwd_stop) {
  fa::arm_kernel_events(fwd_start, fwd_stop, bwd_start, bwd_stop);
  return FA_OK;
}

FA_EXPORT unsigned long long fa_kernel_launches(void) { return fa::g_launches.load(); }

FA_EXPORT unsigned long long fa_scratch_allocs(void) { return fa::scratch_allocs(); }

FA_EXPORT int fa_last_cuda_error(void) { return fa::g_last_cuda_error.load(); }

FA_EXPORT int fa_version(void) { return 100; }

}  // extern "C"
