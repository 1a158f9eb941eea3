// Host-side helpers shared by the C-ABI entry points: TMA tensor-map
// encoding (through the driver entry point, so no -lcuda link is needed),
// device queries and argument checks.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "orthrus.h"

namespace orthrus {

// Encode a bf16 tiled tensor map with 128-byte swizzle.  dims/strides follow
// the driver API (dims[0] innermost; strides in bytes for dims 1..rank-1).
// Returns ORTHRUS_OK, ORTHRUS_ECUDA (entry point missing) or ORTHRUS_EINVAL.
int encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box);

// fp32 tiled tensor map without swizzle (same conventions as above).
int encode_tmap_f32_plain(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                          const uint64_t* strides_bytes, const uint32_t* box);

// Number of SMs of the current device (ORTHRUS_ECUDA on failure).
int current_sm_count(int* sms);

// Raise a kernel's dynamic shared-memory limit on the current device.  Done
// once per (kernel, device) and remembered, so calls made while a stream is
// being captured into a CUDA graph issue no attribute call.
bool opt_in_smem(const void* kernel, int bytes);

// Limit, in nanoseconds, after which a bounded wait inside a kernel gives up
// (passed to every launch; 2 s unless orthrus_set_wait_limit_ns changed it).
uint64_t wait_limit_ns();

// Whether launches carry the programmatic-stream-serialisation attribute
// (on unless the environment variable ORTHRUS_NO_PDL is set when the library
// first launches a kernel).
bool pdl_enabled();

// Whether block attention always launches cooperatively (the environment
// variable ORTHRUS_ATTN_COOPERATIVE is set when the library first launches
// it): for callers that run other kernels concurrently on other streams, so
// the grid starts only once every CTA can be resident.
bool attn_cooperative();

// Launch `kernel` on `s`, with the programmatic-stream-serialisation
// attribute when pdl_enabled(); every kernel of this library calls
// griddepcontrol.wait before it touches memory a preceding kernel may write.
template <typename... KArgs, typename... Args>
int launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                  Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? ORTHRUS_OK : ORTHRUS_ECUDA;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace orthrus
