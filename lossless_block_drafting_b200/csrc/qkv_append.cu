// Block Q/K/V append: the step just before block attention.  The block's keys
// and values go into the scratch slots [L_b, L_b + K) of the shared KV cache
// (gist.science summary of "Orthrus: Memory-Efficient Parallel Token
// Generation via Dual-View Diffusion", technical summary 2.1 and 2.3 item 1:
// both views read and write one cache; the paper's abstract: O(1) overhead),
// after the epilogue of the Qwen3-family projections this build targets: a
// per-head RMS normalisation of q and k, then the rotary position embedding
// with coordinate j paired with j + d/2 and angle (L_b + i) * theta^(-2j/d).
//
// One CTA per (block token, group of 8 heads), one warp per head (a
// Qwen3-8B block of 32 tokens and 48 heads is 192 CTAs): the d/2 angles
// p * theta^(-2j/d) are evaluated in double precision from inverse
// frequencies the host computes once (exact for any position up to 2^31) and
// kept as fp32 (cos, sin) pairs in shared memory; lane l of a warp holds
// elements l, l + 32, ... of its head, so both members of every rotated pair
// sit in the same lane.  The step moves (Hq + 2 Hkv) d bf16 in and out per
// token: latency-bound at decode sizes.
#include <cmath>

#include "common.cuh"
#include "host.h"

namespace orthrus {
namespace qkv {

constexpr int HPB = 8;                  // heads (warps) per CTA
constexpr int THREADS = HPB * 32;
constexpr int MAX_HALF = 64;            // d / 2 for d <= 128

struct Params {
  const __nv_bfloat16* qkv;   // [B*K, (Hq + 2 Hkv) d]
  const __nv_bfloat16* qw;    // [d] or null
  const __nv_bfloat16* kw;    // [d] or null
  __nv_bfloat16* q_out;       // [B, K, Hq, d]
  __nv_bfloat16* kc;          // [B, Hkv, cap, d]
  __nv_bfloat16* vc;
  const int32_t* ctx_lens;
  int32_t* dev_status;
  int K, Hq, Hkv, cap, ngrp;
  float eps;
  double inv_freq[MAX_HALF];  // theta^(-2j/d), j < d/2
};

template <int D>
__global__ void __launch_bounds__(THREADS) qkv_append_kernel(const Params p) {
  constexpr int E = D / 32;  // elements per lane
  __shared__ float2 cs[D / 2];
  grid_dep_launch();
  grid_dep_wait();  // qkv, ctx_lens and the cache may come from the previous kernel
  const int t = blockIdx.x / p.ngrp, grp = blockIdx.x % p.ngrp;
  const int b = t / p.K, i = t - b * p.K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int L = __ldg(p.ctx_lens + b);
  if (L < 0 || L > p.cap - p.K) {
    // same clamping as block attention, so the pair stays consistent
    if (i == 0 && threadIdx.x == 0) report(p.dev_status, ORTHRUS_ECAPACITY);
    L = L < 0 ? 0 : p.cap - p.K;
  }
  const int pos = L + i;
  for (int j = threadIdx.x; j < D / 2; j += THREADS) {
    const double a = static_cast<double>(pos) * p.inv_freq[j];
    double s, c;
    sincos(a, &s, &c);
    cs[j] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
  __syncthreads();
  const int W = p.Hq + 2 * p.Hkv;
  const int hh = grp * HPB + warp;
  if (hh < W) {
    const __nv_bfloat16* src = p.qkv + (static_cast<long long>(t) * W + hh) * D;
    float x[E];
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = __bfloat162float(src[lane + 32 * e]);
    const bool is_q = hh < p.Hq, is_k = !is_q && hh < p.Hq + p.Hkv;
    if (is_q || is_k) {
      const __nv_bfloat16* w = is_q ? p.qw : p.kw;
      if (w != nullptr) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
        const float r = 1.f / sqrtf(ss / D + p.eps);
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] = x[e] * r * __bfloat162float(w[lane + 32 * e]);
      }
#pragma unroll
      for (int e = 0; e < E / 2; ++e) {
        const float2 c = cs[lane + 32 * e];
        const float lo = x[e], hi = x[e + E / 2];
        x[e] = lo * c.x - hi * c.y;
        x[e + E / 2] = hi * c.x + lo * c.y;
      }
    }
    __nv_bfloat16* dst;
    if (is_q) {
      dst = p.q_out + ((static_cast<long long>(b) * p.K + i) * p.Hq + hh) * D;
    } else {
      const int g = is_k ? hh - p.Hq : hh - p.Hq - p.Hkv;
      dst = (is_k ? p.kc : p.vc) +
            ((static_cast<long long>(b) * p.Hkv + g) * p.cap + pos) * D;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) dst[lane + 32 * e] = __float2bfloat16_rn(x[e]);
  }
}

}  // namespace qkv
}  // namespace orthrus

using namespace orthrus;

extern "C" int orthrus_block_qkv_append(const void* qkv, const void* q_norm_w,
                                        const void* k_norm_w, float rope_theta, float rms_eps,
                                        int Hq, int K, const orthrus_kv_cache* cache,
                                        void* q_out, int32_t* dev_status, void* stream) {
  if (qkv == nullptr || cache == nullptr || q_out == nullptr) return ORTHRUS_EINVAL;
  if (K < 1 || Hq < 1 || cache->B < 0 || cache->Hkv < 1) return ORTHRUS_EINVAL;
  if (!(rope_theta > 0.f) || !(rms_eps >= 0.f)) return ORTHRUS_EINVAL;
  if ((q_norm_w == nullptr) != (k_norm_w == nullptr)) return ORTHRUS_EINVAL;
  if (Hq % cache->Hkv != 0) return ORTHRUS_ESHAPE;
  if (cache->d != 64 && cache->d != 128) return ORTHRUS_EUNSUPPORTED;
  if (cache->k == nullptr || cache->v == nullptr || cache->ctx_lens == nullptr)
    return ORTHRUS_EINVAL;
  if (cache->cap < K) return ORTHRUS_ESHAPE;
  if (static_cast<long long>(cache->B) * cache->Hkv * cache->cap >= (1ll << 31) ||
      static_cast<long long>(cache->B) * K >= (1ll << 31))
    return ORTHRUS_EUNSUPPORTED;
  if (!aligned16(qkv) || !aligned16(q_out) || !aligned16(cache->k) || !aligned16(cache->v))
    return ORTHRUS_EALIGN;
  if (cache->B == 0) return ORTHRUS_OK;
  qkv::Params p;
  p.qkv = static_cast<const __nv_bfloat16*>(qkv);
  p.qw = static_cast<const __nv_bfloat16*>(q_norm_w);
  p.kw = static_cast<const __nv_bfloat16*>(k_norm_w);
  p.q_out = static_cast<__nv_bfloat16*>(q_out);
  p.kc = static_cast<__nv_bfloat16*>(cache->k);
  p.vc = static_cast<__nv_bfloat16*>(cache->v);
  p.ctx_lens = cache->ctx_lens;
  p.dev_status = dev_status;
  p.K = K;
  p.Hq = Hq;
  p.Hkv = cache->Hkv;
  p.cap = cache->cap;
  p.eps = rms_eps;
  p.ngrp = (Hq + 2 * cache->Hkv + qkv::HPB - 1) / qkv::HPB;
  for (int j = 0; j < cache->d / 2; ++j)
    p.inv_freq[j] = std::pow(static_cast<double>(rope_theta), -2.0 * j / cache->d);
  const long long nblk = static_cast<long long>(cache->B) * K * p.ngrp;
  if (nblk >= (1ll << 31)) return ORTHRUS_EUNSUPPORTED;
  const dim3 grid(static_cast<unsigned>(nblk));
  const cudaStream_t s = as_stream(stream);
  if (cache->d == 128)
    return launch_kernel(qkv::qkv_append_kernel<128>, grid, dim3(qkv::THREADS), 0, s, p);
  return launch_kernel(qkv::qkv_append_kernel<64>, grid, dim3(qkv::THREADS), 0, s, p);
}
