// Exact consensus and O(1) KV commit, plus a row argmax over given logits.
//
// Method: gist.science summary of "Orthrus: Memory-Efficient Parallel Token
// Generation via Dual-View Diffusion", technical summary 2.3 item 3 (strict
// left-to-right check against the frozen AR head's greedy prediction; on a
// mismatch at index j keep the prefix up to j-1, append the AR correction
// token, shorten the cache); Hacker News thread "Orthrus-Qwen3: ..." post #21
// (accept the longest matching prefix); the paper's abstract (O(1) cache
// overhead).
//
// One warp per sequence: lane i compares position i (K <= 32), a ballot finds
// the first mismatch, lane 0 writes the results and moves the length pointer.
#include "common.cuh"
#include "host.h"

namespace orthrus {
namespace cons {

constexpr int WARPS = 4;

// mode bit 0: verify (argmax/draft -> accept_len/next_tok)
// mode bit 1: commit (accept_len -> ctx_lens)
__global__ void __launch_bounds__(WARPS * 32)
    verify_commit_kernel(const int32_t* __restrict__ argmax, const int32_t* __restrict__ draft,
                         int B, int K, int32_t* accept_len, int32_t* next_tok,
                         int32_t* ctx_lens, int cap, int32_t* dev_status, int mode) {
  grid_dep_launch();
  grid_dep_wait();  // argmax, draft, accept_len and ctx_lens may come from the previous kernel
  const int b = blockIdx.x * WARPS + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  int a;
  if (mode & 1) {
    const long long base = static_cast<long long>(b) * K;
    int am = 0, dr = 0;
    if (lane < K) {
      am = __ldg(argmax + base + lane);
      dr = __ldg(draft + base + lane);
    }
    const unsigned mism = __ballot_sync(0xFFFFFFFFu, lane < K && am != dr);
    a = mism ? __ffs(mism) - 1 : K;
    // correction token: AR choice at the first mismatch; full accept: last draft
    const int src_lane = a < K ? a : K - 1;
    const int am_a = __shfl_sync(0xFFFFFFFFu, am, src_lane);
    const int dr_last = __shfl_sync(0xFFFFFFFFu, dr, K - 1);
    if (lane == 0) {
      accept_len[b] = a;
      next_tok[b] = a < K ? am_a : dr_last;
    }
  } else {
    a = accept_len[b];
  }
  if ((mode & 2) && lane == 0) {
    if (a < 0 || a > K) {
      report(dev_status, ORTHRUS_EINVAL);
      return;
    }
    const long long adv = a + 1 < K ? a + 1 : K;
    long long nl = static_cast<long long>(ctx_lens[b]) + adv;
    if (nl > cap) {
      nl = cap;
      report(dev_status, ORTHRUS_ECAPACITY);
    }
    ctx_lens[b] = static_cast<int32_t>(nl);
  }
}

// Greedy choice over fp32 logits: one block per row, smallest index on ties.
__global__ void __launch_bounds__(256) row_argmax_kernel(const float* __restrict__ logits, int V,
                                                         int32_t* __restrict__ argmax) {
  grid_dep_launch();
  grid_dep_wait();
  const int r = blockIdx.x;
  const float* row = logits + static_cast<long long>(r) * V;
  uint64_t k = 0ull;
  for (int v = threadIdx.x; v < V; v += blockDim.x)
    k = umax64(k, argmax_key(__ldg(row + v), static_cast<uint32_t>(v)));
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) k = umax64(k, shfl_xor_u64(k, m));
  __shared__ uint64_t wbest[8];
  if ((threadIdx.x & 31) == 0) wbest[threadIdx.x >> 5] = k;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) k = umax64(k, wbest[w]);
    argmax[r] = key_index(k);
  }
}

int launch_vc(const int32_t* argmax, const int32_t* draft, int B, int K, int32_t* accept_len,
              int32_t* next_tok, int32_t* ctx_lens, int cap, int32_t* dev_status, int mode,
              void* stream) {
  if (B == 0) return ORTHRUS_OK;
  const int blocks = (B + WARPS - 1) / WARPS;
  return launch_kernel(verify_commit_kernel, dim3(blocks), dim3(WARPS * 32), 0, as_stream(stream),
                       argmax, draft, B, K, accept_len, next_tok, ctx_lens, cap, dev_status,
                       mode);
}

}  // namespace cons
}  // namespace orthrus

using namespace orthrus;

extern "C" int orthrus_verify(const int32_t* argmax, const int32_t* draft, int B, int K,
                              int32_t* accept_len, int32_t* next_tok, void* stream) {
  if (B < 0 || K < 1 || K > 32) return ORTHRUS_EINVAL;
  if (B > 0 && (argmax == nullptr || draft == nullptr || accept_len == nullptr ||
                next_tok == nullptr))
    return ORTHRUS_EINVAL;
  return cons::launch_vc(argmax, draft, B, K, accept_len, next_tok, nullptr, 0, nullptr, 1,
                         stream);
}

extern "C" int orthrus_kv_commit(const orthrus_kv_cache* cache, const int32_t* accept_len, int K,
                                 int32_t* dev_status, void* stream) {
  if (cache == nullptr || K < 1 || K > 32) return ORTHRUS_EINVAL;
  if (cache->B < 0 || cache->cap < 0) return ORTHRUS_EINVAL;
  if (cache->B > 0 && (cache->ctx_lens == nullptr || accept_len == nullptr))
    return ORTHRUS_EINVAL;
  return cons::launch_vc(nullptr, nullptr, cache->B, K, const_cast<int32_t*>(accept_len),
                         nullptr, cache->ctx_lens, cache->cap, dev_status, 2, stream);
}

extern "C" int orthrus_verify_commit(const int32_t* argmax, const int32_t* draft, int B, int K,
                                     int32_t* accept_len, int32_t* next_tok,
                                     const orthrus_kv_cache* cache, int32_t* dev_status,
                                     void* stream) {
  if (cache == nullptr || B < 0 || K < 1 || K > 32) return ORTHRUS_EINVAL;
  if (cache->B != B) return ORTHRUS_ESHAPE;
  if (cache->cap < 0) return ORTHRUS_EINVAL;
  if (B > 0 && (argmax == nullptr || draft == nullptr || accept_len == nullptr ||
                next_tok == nullptr || cache->ctx_lens == nullptr))
    return ORTHRUS_EINVAL;
  return cons::launch_vc(argmax, draft, B, K, accept_len, next_tok, cache->ctx_lens, cache->cap,
                         dev_status, 3, stream);
}

extern "C" int orthrus_row_argmax_f32(const float* logits, int R, int V, int32_t* argmax,
                                      void* stream) {
  if (R < 0 || V < 1) return ORTHRUS_EINVAL;
  if (R > 0 && (logits == nullptr || argmax == nullptr)) return ORTHRUS_EINVAL;
  if (R == 0) return ORTHRUS_OK;
  return launch_kernel(cons::row_argmax_kernel, dim3(R), dim3(256), 0, as_stream(stream), logits,
                       V, argmax);
}
