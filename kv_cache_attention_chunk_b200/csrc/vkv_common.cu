// Host helpers shared by the entry points: device checks, TMA descriptor
// encoding (through the driver entry point, so the library loads on machines
// without a GPU driver), status strings.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "vkv_internal.h"
#include "vkv_tmap.h"

namespace vkv {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

struct DevInfo {
  int checked = 0;  // 0 unknown, 1 usable, -1 unusable
  int sms = 0;
};
constexpr int kMaxDevices = 64;
DevInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

void init_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}
}  // namespace

int device_sm_count(int* dev_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return -1;
  }
  if (dev_out) *dev_out = dev;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& di = g_dev[dev];
  if (di.checked == 0) {
    int major = 0, minor = 0, sms = 0;
    bool ok = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
              cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
              cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
    // the kernels are built for sm_100a only
    di.checked = (ok && major == 10 && minor == 0 && sms > 0) ? 1 : -1;
    di.sms = sms;
    cudaGetLastError();
  }
  return di.checked == 1 ? di.sms : -1;
}

bool encode_tmap_bf16_4d(CUtensorMap* tm, const void* ptr, const uint64_t dims[4],
                         const uint64_t strides_bytes[3], const uint32_t box[4]) {
  return encode_tmap_bf16_4d_swizzle(tm, ptr, dims, strides_bytes, box, 128);
}

bool encode_tmap_bf16_4d_swizzle(CUtensorMap* tm, const void* ptr, const uint64_t dims[4],
                                 const uint64_t strides_bytes[3], const uint32_t box[4], int swizzle_bytes) {
  std::call_once(g_encode_once, init_encode);
  if (!g_encode) return false;
  cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gs[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
  cuuint32_t bd[4] = {box[0], box[1], box[2], box[3]};
  cuuint32_t es[4] = {1, 1, 1, 1};
  if (swizzle_bytes != 128 && swizzle_bytes != 64) return false;
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), gd, gs, bd, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

#ifdef VKV_TEST_AIDS
namespace {
std::atomic<int> g_withhold{0};
}  // namespace

bool take_withhold_request() {
  int n = g_withhold.load();
  while (n > 0) {
    if (g_withhold.compare_exchange_weak(n, n - 1)) return true;
  }
  return false;
}
#endif

bool tensor_aligned(const vkv_tensor& t) {
  return (reinterpret_cast<uintptr_t>(t.ptr) & 15u) == 0 && (t.sb % 8) == 0 && (t.st % 8) == 0 &&
         (t.sh % 8) == 0;
}

}  // namespace vkv

extern "C" const char* vkv_status_string(vkv_status s) {
  switch (s) {
    case VKV_OK: return "ok";
    case VKV_ERR_NULL: return "a required pointer is NULL";
    case VKV_ERR_SHAPE: return "a size is out of range or sizes disagree";
    case VKV_ERR_ALIGN: return "a pointer or stride breaks the 16-byte rule";
    case VKV_ERR_RANGE: return "a segment or offset lies outside the cache";
    case VKV_ERR_UNSUPPORTED: return "request outside what this build implements";
    case VKV_ERR_CUDA: return "no usable sm_100 device, or a CUDA call failed";
    case VKV_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

extern "C" int32_t vkv_version(void) { return 300; }

extern "C" int32_t vkv_abi_sizeof(int32_t which) {
  switch (which) {
    case 0: return (int32_t)sizeof(vkv_attn_args);
    case 1: return (int32_t)sizeof(vkv_select_args);
    case 2: return (int32_t)sizeof(vkv_tensor);
    case 3: return (int32_t)sizeof(vkv_segment);
    case 4: return (int32_t)sizeof(vkv_compact_args);
    case 5: return (int32_t)sizeof(vkv_head_rule);
    case 6: return (int32_t)sizeof(vkv_persist_args);
    case 7: return (int32_t)sizeof(vkv_latent_args);
    case 8: return (int32_t)sizeof(vkv_schedule);
  }
  return -1;
}

#ifdef VKV_TEST_AIDS
// Test build only (vkv_test.h).
extern "C" vkv_status vkv_debug_withhold_copy(int32_t n_calls) {
  if (n_calls < 0) return VKV_ERR_SHAPE;
  vkv::g_withhold.store(n_calls);
  return VKV_OK;
}
#endif
