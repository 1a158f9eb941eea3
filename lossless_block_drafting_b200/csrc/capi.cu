// C-ABI plumbing: status strings, ABI version, tensor-map encoding and device
// queries shared by the kernels' host launchers.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdlib>
#include <mutex>

#include "host.h"

namespace orthrus {

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

void resolve_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q{};
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess) {
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
}
}  // namespace

namespace {
int encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, CUtensorMapSwizzle swizzle,
                const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                const uint32_t* box) {
  std::call_once(g_encode_once, resolve_encode);
  if (g_encode == nullptr) return ORTHRUS_ECUDA;
  cuuint64_t gdim[5];
  cuuint64_t gstride[4];
  cuuint32_t bdim[5];
  cuuint32_t estride[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bdim[i] = box[i];
    estride[i] = 1;
    if (i + 1 < rank) gstride[i] = strides_bytes[i];
  }
  CUresult r = g_encode(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base), gdim,
                        gstride, bdim, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? ORTHRUS_OK : ORTHRUS_EINVAL;
}
}  // namespace

int encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_128B, base, rank,
                     dims, strides_bytes, box);
}

int encode_tmap_f32_plain(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                          const uint64_t* strides_bytes, const uint32_t* box) {
  return encode_tmap(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_SWIZZLE_NONE, base, rank,
                     dims, strides_bytes, box);
}

bool opt_in_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static const void* done_kernel[64][8] = {};
  static int done_bytes[64][8] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < 8; ++i)
    if (done_kernel[dev][i] == kernel && done_bytes[dev][i] >= bytes) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  for (int i = 0; i < 8; ++i)
    if (done_kernel[dev][i] == nullptr || done_kernel[dev][i] == kernel) {
      done_kernel[dev][i] = kernel;
      done_bytes[dev][i] = bytes;
      break;
    }
  return true;
}

namespace {
constexpr uint64_t kDefaultWaitNs = 2000000000ull;  // 2 s
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
}  // namespace

uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

bool pdl_enabled() {
  static const bool on = std::getenv("ORTHRUS_NO_PDL") == nullptr;
  return on;
}

bool attn_cooperative() {
  static const bool on = std::getenv("ORTHRUS_ATTN_COOPERATIVE") != nullptr;
  return on;
}

int current_sm_count(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ORTHRUS_ECUDA;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return ORTHRUS_ECUDA;
  return ORTHRUS_OK;
}

}  // namespace orthrus

extern "C" const char* orthrus_status_str(int status) {
  switch (status) {
    case ORTHRUS_OK: return "ORTHRUS_OK";
    case ORTHRUS_EINVAL: return "ORTHRUS_EINVAL: invalid argument";
    case ORTHRUS_ESHAPE: return "ORTHRUS_ESHAPE: inconsistent shapes";
    case ORTHRUS_EUNSUPPORTED: return "ORTHRUS_EUNSUPPORTED: unsupported configuration";
    case ORTHRUS_ECUDA: return "ORTHRUS_ECUDA: CUDA call failed";
    case ORTHRUS_ECAPACITY: return "ORTHRUS_ECAPACITY: KV cache capacity exceeded";
    case ORTHRUS_EWORKSPACE: return "ORTHRUS_EWORKSPACE: workspace missing or too small";
    case ORTHRUS_EALIGN: return "ORTHRUS_EALIGN: pointer not 16-byte aligned";
    case ORTHRUS_ETIMEOUT: return "ORTHRUS_ETIMEOUT: bounded device wait gave up";
    default: return "ORTHRUS: unknown status";
  }
}

extern "C" int orthrus_abi_version(void) { return 3; }

extern "C" int orthrus_set_wait_limit_ns(uint64_t ns) {
  orthrus::g_wait_ns.store(ns == 0 ? orthrus::kDefaultWaitNs : ns, std::memory_order_relaxed);
  return ORTHRUS_OK;
}
