// Status strings, the per-device error flag, SM-count cache and TMA
// descriptor encoding for libpagedattn.
#include <map>
#include <mutex>
#include <utility>

#include "pa_host.h"

// One int per device that loads the library; kernels OR PA_DEVERR_* bits into it.
static __device__ int g_pa_device_error = 0;

namespace pa {

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_err_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
thread_local int g_last_launches = 0;
thread_local int g_test_kind = 0;            // pa_testing_wait_fault: kernel kind, one-shot
thread_local long long g_test_limit = 0;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int current_device() {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
  return d;
}
}  // namespace

int* device_error_flag() {
  const int d = current_device();
  if (d < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[d]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_pa_device_error) != cudaSuccess) {
      (void)cudaGetLastError();  // reported by this call's status, not a later launch check
      return nullptr;
    }
    g_err_ptr[d] = static_cast<int*>(p);
  }
  return g_err_ptr[d];
}

int* launch_prologue() {
  (void)cudaGetLastError();
  return device_error_flag();
}

int num_sms() {
  const int d = current_device();
  if (d < 0) return 0;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sms[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) return 0;
    g_sms[d] = n;
  }
  return g_sms[d];
}

bool ensure_dynamic_smem(const void* func, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> granted;
  const int d = current_device();
  if (d < 0) return false;
  std::lock_guard<std::mutex> lk(mu);
  int& have = granted[{func, d}];
  if (have >= bytes) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  have = bytes;
  return true;
}

static bool load_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  return true;
}

bool encode_tmap(CUtensorMap* out, CUtensorMapDataType type, const void* base, int rank,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle) {
  if (!load_encoder() || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides_bytes[i];
  }
  CUresult r = g_encode(out, type, rank, const_cast<void*>(base), d, st, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_16bit(CUtensorMap* out, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle) {
  return encode_tmap(out, CU_TENSOR_MAP_DATA_TYPE_UINT16, base, rank, dims, strides_bytes, box,
                     swizzle);
}


long long take_wait_limit(int kind, int* withhold) {
  *withhold = 0;
  if (g_test_kind != kind) return kWaitLimitCycles;
  *withhold = 1;
  const long long lim = g_test_limit;
  g_test_kind = 0;
  return lim;
}

void set_launch_count(int n) { g_last_launches = n; }
int launch_count() { return g_last_launches; }

}  // namespace pa

extern "C" {

const char* pa_status_string(int s) {
  switch (s) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_WORKSPACE_TOO_SMALL: return "PA_ERR_WORKSPACE_TOO_SMALL";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_DEVICE_DATA: return "PA_ERR_DEVICE_DATA";
    default: return "PA_ERR_UNKNOWN";
  }
}

pa_status pa_get_device_error(void* stream, int32_t* code) {
  if (!code) return PA_ERR_INVALID_ARG;
  *code = 0;
  int* flag = pa::device_error_flag();
  if (!flag) return PA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, flag, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaMemsetAsync(flag, 0, sizeof(int), s) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  *code = v;
  return v ? PA_ERR_DEVICE_DATA : PA_OK;
}

int pa_last_launch_count(void) { return pa::g_last_launches; }

pa_status pa_testing_wait_fault(int kernel, long long wait_limit_cycles) {
  if (kernel < 0 || kernel > 2 || (kernel != 0 && wait_limit_cycles <= 0))
    return PA_ERR_INVALID_ARG;
  pa::g_test_kind = kernel;
  pa::g_test_limit = wait_limit_cycles;
  return PA_OK;
}

}  // extern "C"
