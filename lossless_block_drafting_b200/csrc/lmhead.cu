// LM head with the greedy (argmax) choice fused into the GEMM epilogue.
//
// Method: gist.science summary of "Orthrus: Memory-Efficient Parallel Token
// Generation via Dual-View Diffusion", technical summary 2.3 items 2-3: the
// frozen AR head scores all K block positions in one pass and a drafted token
// survives only if it equals that head's greedy prediction.  So the step needs
// argmax_v (h_r . W_v) per row r, not the logits.
//
// Design (B200, sm_100a).  Swap-AB tcgen05 GEMM: the vocabulary supplies the
// 128-row M dimension (W tile, K-major), the R = B*K hidden rows the N
// dimension (h, K-major, N padded to a multiple of 32), fp32 accumulators in
// TMEM.  Each CTA of a one-per-SM grid owns an equal, 16-row-granular slice of
// the vocabulary; it streams W through a TMA ring (64 hidden elements = one
// 128-byte swizzled row per stage, evict-first L2 policy) and keeps two to
// four tiles' accumulators live at once so each h chunk is fetched once per
// two to four W tiles.  While two rounds fit in TMEM (N <= 128) the
// accumulators are double-buffered so the epilogue of one round overlaps the
// MMAs of the next.  The epilogue (one thread per vocab row) maps
// each logit to a 64-bit key (order-preserving value bits | inverted index,
// so ties go to the smallest index), reduces across the warp with a
// transposing butterfly, and keeps a per-warp best per column in shared
// memory.  A tiny second kernel reduces the per-CTA bests.  Logits never
// reach HBM.
#include <cuda_bf16.h>

#include <mutex>

#include "common.cuh"
#include "host.h"

namespace orthrus {
namespace lmh {

constexpr int BM = 128;       // vocab rows per tile (tcgen05 M)
constexpr int BK = 64;        // hidden elements per stage (one 128-byte row)
constexpr int GROUP = 16;     // vocabulary partition granularity (rows)
constexpr int THREADS = 256;
constexpr int MAX_PASS_ROWS = 256;
constexpr int W_TILE_BYTES = BM * 128;  // 16 KB
constexpr int SMEM_LIMIT = 232448;      // 227 KB opt-in maximum per block

struct Params {
  uint64_t* part_keys;  // [gridDim.x][Npad]
  int32_t* dev_status;
  unsigned long long wait_ns;  // bounded-wait limit
  int R, Npad, H, V, TPR, NB, NS, stage_bytes;
};

struct Plan {
  int Npad, TPR, NB, NS, stage_bytes, smem;
};

// Tiles per round TPR: every h chunk staged feeds TPR W tiles, so the
// shared-memory fill per MMA shrinks as TPR grows (at N = 256 one tile per
// stage would need about 96 B/clk per SM, two tiles 64 B/clk).  The round's
// accumulators are double-buffered (NB = 2) while 2 * TPR * Npad fits the 512
// TMEM columns; otherwise (Npad > 128) a single buffer holds two tiles and
// the MMAs of the next round wait for the epilogue.
inline Plan make_plan(int R) {
  Plan pl;
  pl.Npad = ((R + 31) / 32) * 32;
  const int tpr = MAX_PASS_ROWS / pl.Npad;
  pl.TPR = tpr < 2 ? 2 : (tpr > 4 ? 4 : tpr);
  pl.NB = 2 * pl.TPR * pl.Npad <= 512 ? 2 : 1;
  pl.stage_bytes = pl.TPR * W_TILE_BYTES + pl.Npad * 128;
  const int fixed = 1024 /*align*/ + 4 * pl.Npad * 8 /*bests*/ + 64 * 8 /*barriers*/ + 16;
  pl.NS = (SMEM_LIMIT - fixed) / pl.stage_bytes;
  if (pl.NS > 8) pl.NS = 8;
  pl.smem = fixed + pl.NS * pl.stage_bytes;
  return pl;
}

__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity, int32_t* status) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) {  // 200 ms
      report(status, ORTHRUS_ETIMEOUT);
      return;
    }
  }
}

// Rows of tile t of a CTA's vocabulary slice [row0, row_end).
__device__ __forceinline__ int tile_rows_of(int row0, int row_end, int t) {
  const int a = row0 + t * BM;
  const int e = a + BM < row_end ? a + BM : row_end;
  return e - a;
}

// 32 keys per lane -> lane l holds the warp-wide max of column l.
__device__ __forceinline__ uint64_t transpose_max(uint64_t (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int k = 0; k < s; ++k) {
      const uint64_t send = upper ? v[k] : v[k + s];
      const uint64_t keep = upper ? v[k + s] : v[k];
      v[k] = umax64(keep, shfl_xor_u64(send, s));
    }
  }
  return v[0];
}

template <bool kShortWait>
__global__ void __launch_bounds__(THREADS, 1)
    lmhead_argmax_kernel(const __grid_constant__ CUtensorMap tmW128,
                         const __grid_constant__ CUtensorMap tmW16,
                         const __grid_constant__ CUtensorMap tmH, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sb0 = raw_addr + pad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int NS = p.NS, TPR = p.TPR, Npad = p.Npad;
  const int off_best = NS * p.stage_bytes;
  const int off_bar = off_best + 4 * Npad * 8;
  const uint32_t bar = sb0 + off_bar;
  auto full = [&](int s) { return bar + 8u * s; };
  auto empty = [&](int s) { return bar + 8u * (NS + s); };
  auto acc_full = [&](int i) { return bar + 8u * (2 * NS + i); };
  auto acc_free = [&](int i) { return bar + 8u * (2 * NS + 2 + i); };
  const uint32_t mma_done = bar + 8u * (2 * NS + 4);
  uint64_t* best = reinterpret_cast<uint64_t*>(smem + off_best);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + off_bar + 8 * (2 * NS + 5));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int NB = p.NB;
  const uint32_t tmem_cols = (NB * TPR * Npad) <= 256 ? 256u : 512u;

  // This CTA's vocabulary slice, in 16-row groups.
  const long long NG = (p.V + GROUP - 1) / GROUP;
  const long long g0 = static_cast<long long>(blockIdx.x) * NG / gridDim.x;
  const long long g1 = static_cast<long long>(blockIdx.x + 1) * NG / gridDim.x;
  const int row0 = static_cast<int>(g0 * GROUP);
  const int row_end = static_cast<int>(g1 * GROUP < p.V ? g1 * GROUP : p.V);
  const int n_rows = row_end > row0 ? row_end - row0 : 0;
  const int n_tiles = (n_rows + BM - 1) / BM;
  const int n_rounds = (n_tiles + TPR - 1) / TPR;
  const int n_k = p.H / BK;

  // Programmatic dependent launch: the prologue below (barriers, TMEM) overlaps
  // the previous kernel's tail; h and the workspace are touched only after
  // grid_dep_wait.
  grid_dep_launch();
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_free(i), 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmW128);
  }
  for (int i = threadIdx.x; i < 4 * Npad; i += THREADS) best[i] = 0ull;
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  grid_dep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto tile_rows = [&](int t) { return tile_rows_of(row0, row_end, t); };

#define WAIT_OR(barrier, parity, on_fail) \
  if (!mbar_wait_bounded<kShortWait>((barrier), (parity), abort_flag, p.dev_status, p.wait_ns)) on_fail
#define WARP_WAIT_OR(barrier, parity, on_fail) \
  if (!mbar_wait_warp<kShortWait>((barrier), (parity), abort_flag, p.dev_status, p.wait_ns)) on_fail

  if (n_tiles > 0 && warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    prefetch_tmap(&tmW128);
    prefetch_tmap(&tmW16);
    prefetch_tmap(&tmH);
    const uint64_t policy = policy_evict_first();
    int it = 0;
    bool ok = true;
    for (int q = 0; ok && q < n_rounds; ++q) {
      const int t0 = q * TPR;
      const int ntr = n_tiles - t0 < TPR ? n_tiles - t0 : TPR;
      uint32_t bytes = static_cast<uint32_t>(Npad) * 128u;
      for (int u = 0; u < ntr; ++u) {
        const int rows = tile_rows(t0 + u);
        bytes += (rows == BM ? BM : ((rows + GROUP - 1) / GROUP) * GROUP) * 128u;
      }
      for (int kc = 0; kc < n_k; ++kc, ++it) {
        const int stage = it % NS;
        WAIT_OR(empty(stage), ((it / NS) & 1) ^ 1, { ok = false; break; });
        mbar_arrive_expect_tx(full(stage), bytes);
        const uint32_t sbase = sb0 + stage * p.stage_bytes;
        for (int u = 0; u < ntr; ++u) {
          const int tr0 = row0 + (t0 + u) * BM;
          const int rows = tile_rows(t0 + u);
          const uint32_t dst = sbase + u * W_TILE_BYTES;
          if (rows == BM) {
            tma_load_2d_hint(dst, &tmW128, full(stage), kc * BK, tr0, policy);
          } else {
            for (int z = 0; z * GROUP < rows; ++z)
              tma_load_2d_hint(dst + z * GROUP * 128, &tmW16, full(stage), kc * BK,
                               tr0 + z * GROUP, policy);
          }
        }
        tma_load_2d(sbase + TPR * W_TILE_BYTES, &tmH, full(stage), kc * BK, 0);
      }
    }
    for (int j = (it > NS ? it - NS : 0); j < it; ++j) mbar_wait_drain(full(j % NS), (j / NS) & 1, p.dev_status);
  } else if (n_tiles > 0 && warp == 1 && lane == 0) {
    // -------------------------------------------------------- MMA issuer
    const uint32_t idesc = make_idesc_bf16_f32(BM, Npad, false, false);
    int it = 0;
    bool ok = true;
    for (int q = 0; ok && q < n_rounds; ++q) {
      const int buf = q % NB;
      const int ntr = n_tiles - q * TPR < TPR ? n_tiles - q * TPR : TPR;
      if (q >= NB) {
        WAIT_OR(acc_free(buf), ((q - NB) / NB) & 1, break);
      }
      tc_fence_after();
      const uint32_t acc = tmem + static_cast<uint32_t>(buf * TPR * Npad);
      for (int kc = 0; kc < n_k; ++kc, ++it) {
        const int stage = it % NS;
        WAIT_OR(full(stage), (it / NS) & 1, { ok = false; break; });
        tc_fence_after();
        const uint32_t sbase = sb0 + stage * p.stage_bytes;
        const uint32_t hbase = sbase + TPR * W_TILE_BYTES;
        for (int u = 0; u < ntr; ++u) {
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad =
                make_sdesc(sbase + u * W_TILE_BYTES + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = make_sdesc(hbase + kk * 32, 16, 1024, kSwizzle128B);
            mma_bf16_ss(acc + u * Npad, ad, bd, idesc, (kc | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit(empty(stage));
      }
      if (ok) mma_commit(acc_full(buf));
    }
    mma_commit(mma_done);
    mbar_wait_drain(mma_done, 0, p.dev_status);
  } else if (warp >= 4) {
    // --------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint64_t* my_best = best + quarter * Npad;
    for (int q = 0; q < n_rounds; ++q) {
      const int buf = q % NB;
      const int ntr = n_tiles - q * TPR < TPR ? n_tiles - q * TPR : TPR;
      WARP_WAIT_OR(acc_full(buf), (q / NB) & 1, break);
      tc_fence_after();
      for (int u = 0; u < ntr; ++u) {
        const int t = q * TPR + u;
        const int v = row0 + t * BM + quarter * 32 + lane;
        const bool valid = (t * BM + quarter * 32 + lane) < n_rows;
        for (int cc = 0; cc < Npad; cc += 32) {
          uint32_t raw[32];
          tmem_ld32(lane_base + static_cast<uint32_t>(buf * TPR * Npad + u * Npad + cc), raw);
          tmem_wait_ld();
          uint64_t key[32];
#pragma unroll
          for (int k = 0; k < 32; ++k)
            key[k] = valid ? argmax_key(__uint_as_float(raw[k]), static_cast<uint32_t>(v)) : 0ull;
          const uint64_t m = transpose_max(key, lane);
          my_best[cc + lane] = umax64(my_best[cc + lane], m);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_free(buf));
    }
    // Merge the four warps' bests and publish this CTA's candidates.
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int t = threadIdx.x - 128;
    for (int col = t; col < Npad; col += 128) {
      uint64_t k = best[col];
      for (int w = 1; w < 4; ++w) k = umax64(k, best[w * Npad + col]);
      p.part_keys[static_cast<long long>(blockIdx.x) * Npad + col] = k;
    }
  }
#undef WAIT_OR
#undef WARP_WAIT_OR

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// Reduce the per-CTA candidates of each row; one block per row.
__global__ void __launch_bounds__(256) lmhead_reduce_kernel(const uint64_t* __restrict__ keys,
                                                            int n_ctas, int Npad,
                                                            int32_t* __restrict__ argmax,
                                                            float* __restrict__ max_logit) {
  grid_dep_launch();
  grid_dep_wait();  // the candidate keys come from the main kernel
  const int r = blockIdx.x;
  uint64_t k = 0ull;
  for (int c = threadIdx.x; c < n_ctas; c += blockDim.x)
    k = umax64(k, __ldcg(keys + static_cast<long long>(c) * Npad + r));
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) k = umax64(k, shfl_xor_u64(k, m));
  __shared__ uint64_t wbest[8];
  if ((threadIdx.x & 31) == 0) wbest[threadIdx.x >> 5] = k;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) k = umax64(k, wbest[w]);
    argmax[r] = key_index(k);
    if (max_logit != nullptr) max_logit[r] = k == 0ull ? __int_as_float(0x7fc00000) : key_value(k);
  }
}

}  // namespace lmh
}  // namespace orthrus

using namespace orthrus;

extern "C" int orthrus_lmhead_workspace_size(int R, int V, size_t* bytes) {
  if (bytes == nullptr || R < 0 || V < 1) return ORTHRUS_EINVAL;
  int sms = 0;
  const int rc = current_sm_count(&sms);
  if (rc != ORTHRUS_OK) return rc;
  *bytes = static_cast<size_t>(sms) * lmh::MAX_PASS_ROWS * sizeof(uint64_t) + 256;
  return ORTHRUS_OK;
}

extern "C" int orthrus_lmhead_argmax(const void* h, const void* W, int R, int H, int V,
                                     int32_t* argmax, float* max_logit, void* workspace,
                                     size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (h == nullptr || W == nullptr || argmax == nullptr) return ORTHRUS_EINVAL;
  if (R < 0 || V < 1 || H < lmh::BK) return ORTHRUS_EINVAL;
  if (H % lmh::BK != 0) return ORTHRUS_EUNSUPPORTED;
  if (!aligned16(h) || !aligned16(W) || !aligned16(workspace)) return ORTHRUS_EALIGN;
  if (R == 0) return ORTHRUS_OK;
  int sms = 0;
  int rc = current_sm_count(&sms);
  if (rc != ORTHRUS_OK) return rc;
  if (workspace == nullptr || ws_bytes < static_cast<size_t>(sms) * lmh::MAX_PASS_ROWS * 8 + 256)
    return ORTHRUS_EWORKSPACE;
  const cudaStream_t s = as_stream(stream);

  CUtensorMap tw128, tw16;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(H), static_cast<uint64_t>(V)};
    const uint64_t strides[1] = {static_cast<uint64_t>(H) * 2};
    const uint32_t box128[2] = {64u, 128u};
    const uint32_t box16[2] = {64u, 16u};
    rc = encode_tmap_bf16(&tw128, W, 2, dims, strides, box128);
    if (rc != ORTHRUS_OK) return rc;
    rc = encode_tmap_bf16(&tw16, W, 2, dims, strides, box16);
    if (rc != ORTHRUS_OK) return rc;
  }
  const uint64_t wait_ns = wait_limit_ns();
  auto* kfn = wait_ns < kShortWaitNs ? lmh::lmhead_argmax_kernel<true>
                                     : lmh::lmhead_argmax_kernel<false>;
  if (!opt_in_smem(reinterpret_cast<const void*>(kfn), lmh::SMEM_LIMIT)) return ORTHRUS_ECUDA;
  const int grid = static_cast<int>((static_cast<long long>(V) + lmh::GROUP - 1) / lmh::GROUP <
                                            sms
                                        ? (V + lmh::GROUP - 1) / lmh::GROUP
                                        : sms);
  uint64_t* keys = static_cast<uint64_t*>(workspace);
  for (int r0 = 0; r0 < R; r0 += lmh::MAX_PASS_ROWS) {
    const int Rp = R - r0 < lmh::MAX_PASS_ROWS ? R - r0 : lmh::MAX_PASS_ROWS;
    const lmh::Plan pl = lmh::make_plan(Rp);
    CUtensorMap th;
    const uint64_t dims[2] = {static_cast<uint64_t>(H), static_cast<uint64_t>(Rp)};
    const uint64_t strides[1] = {static_cast<uint64_t>(H) * 2};
    const uint32_t box[2] = {64u, static_cast<uint32_t>(pl.Npad)};
    rc = encode_tmap_bf16(&th, static_cast<const __nv_bfloat16*>(h) + static_cast<size_t>(r0) * H,
                          2, dims, strides, box);
    if (rc != ORTHRUS_OK) return rc;
    lmh::Params p;
    p.part_keys = keys;
    p.dev_status = dev_status;
    p.wait_ns = wait_ns;
    p.R = Rp;
    p.Npad = pl.Npad;
    p.H = H;
    p.V = V;
    p.TPR = pl.TPR;
    p.NB = pl.NB;
    p.NS = pl.NS;
    p.stage_bytes = pl.stage_bytes;
    rc = launch_kernel(kfn, dim3(grid), dim3(lmh::THREADS),
                       static_cast<size_t>(pl.smem), s, tw128, tw16, th, p);
    if (rc != ORTHRUS_OK) return rc;
    rc = launch_kernel(lmh::lmhead_reduce_kernel, dim3(Rp), dim3(256), 0, s,
                       static_cast<const uint64_t*>(keys), grid, pl.Npad, argmax + r0,
                       max_logit ? max_logit + r0 : static_cast<float*>(nullptr));
    if (rc != ORTHRUS_OK) return rc;
  }
  return ORTHRUS_OK;
}

// ---------------------------------------------------------------------------
// LM head + argmax without any device allocation by the caller.
//
// Some callers cannot hand this library a workspace: a plain C or embedded
// host program that links only this library and has no device allocator of
// its own, a serving loop whose memory plan is frozen after start-up (where a
// cudaMalloc could fail under fragmentation or stall every stream, because it
// synchronises the device), or a runtime that owns all device memory and does
// not lend scratch to its kernels.  For them this entry point keeps the
// per-CTA candidate keys in a fixed array in the library's own device memory
// instead of a caller workspace.
//
//   * The array holds kNoAllocMaxCtas * 256 candidate keys plus the 256-byte
//     tail the workspace entry point asks for (512.25 KB).  It lives in every
//     GPU that loads the library, for as long as the process runs.
//   * All calls share it and it keeps the last call's contents.  Nothing in it
//     needs to start at zero: every CTA overwrites all of its keys before the
//     reduction reads them.  Calls whose kernels overlap on the GPU (other
//     streams, other host threads) race on the array; order them on one
//     stream.
//   * The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress) and remembers it.  That query is not a stream
//     operation; make the first call on a device before any stream capture.
//   * A device with more SMs than kNoAllocMaxCtas is rejected with
//     ORTHRUS_EWORKSPACE before anything is launched.
// The kernels and their arguments are exactly those of orthrus_lmhead_argmax.
namespace orthrus {
namespace lmh {

constexpr int kNoAllocMaxCtas = 256;
// Exactly what orthrus_lmhead_workspace_size asks for on a kNoAllocMaxCtas-SM
// device: kNoAllocMaxCtas * MAX_PASS_ROWS keys and 256 bytes more.
static __device__ __align__(256) uint64_t g_noalloc_keys[kNoAllocMaxCtas * MAX_PASS_ROWS + 32];
static_assert(sizeof(g_noalloc_keys) ==
                  static_cast<size_t>(kNoAllocMaxCtas) * MAX_PASS_ROWS * sizeof(uint64_t) + 256,
              "no-alloc scratch must cover the workspace size at the largest SM count");

// Device address of g_noalloc_keys on the current device (looked up once per
// device; the symbol's host-side name is only a handle, never a pointer the
// kernel may use).
int noalloc_scratch(uint64_t** out) {
  static std::mutex mu;
  static uint64_t* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ORTHRUS_ECUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_keys) != cudaSuccess || p == nullptr)
      return ORTHRUS_ECUDA;
    addr[dev] = static_cast<uint64_t*>(p);
  }
  *out = addr[dev];
  return ORTHRUS_OK;
}

}  // namespace lmh
}  // namespace orthrus

extern "C" int orthrus_lmhead_argmax_noalloc(const void* h, const void* W, int R, int H, int V,
                                             int32_t* argmax, float* max_logit,
                                             int32_t* dev_status, void* stream) {
  if (h == nullptr || W == nullptr || argmax == nullptr) return ORTHRUS_EINVAL;
  if (R < 0 || V < 1 || H < lmh::BK) return ORTHRUS_EINVAL;
  if (H % lmh::BK != 0) return ORTHRUS_EUNSUPPORTED;
  if (!aligned16(h) || !aligned16(W)) return ORTHRUS_EALIGN;
  if (R == 0) return ORTHRUS_OK;
  int sms = 0;
  int rc = current_sm_count(&sms);
  if (rc != ORTHRUS_OK) return rc;
  if (sms > lmh::kNoAllocMaxCtas) return ORTHRUS_EWORKSPACE;
  uint64_t* scratch = nullptr;
  rc = lmh::noalloc_scratch(&scratch);
  if (rc != ORTHRUS_OK) return rc;
  return orthrus_lmhead_argmax(h, W, R, H, V, argmax, max_logit, scratch,
                               sizeof(lmh::g_noalloc_keys), dev_status, stream);
}
