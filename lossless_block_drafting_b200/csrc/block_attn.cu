// Block-query attention over the shared KV cache, both Orthrus mask modes.
//
// Method: gist.science summary of "Orthrus: Memory-Efficient Parallel Token
// Generation via Dual-View Diffusion", technical summary 2.1 (both views read
// one KV cache), 2.2 (M_diff: causal context + bidirectional block), 2.3 items
// 1-2 (diffusion pass over anchor + K-1 masks; AR pass verifies all K
// positions at once).  Block row i of sequence b sees keys [0, L_b + K) in
// diffusion mode and [0, L_b + i + 1) in AR mode.
//
// Design (B200, sm_100a).  One KV head serves G = Hq/Hkv query heads, so the
// G*K queries of a (sequence, KV head) pair are packed into one 128-row tile
// (row r = i*Gc + hh) and every K/V byte is read from HBM once.  The work of
// all (sequence, KV head) segments is cut into 64-key tiles and spread evenly
// over a persistent grid of one CTA per SM (split-KV / flash-decoding); a
// CTA's contiguous tile range may cross segment boundaries and then emits one
// partial result per segment piece.  Per CTA (12 warps), each single-thread
// role on its own ring so no wait of one stream stalls another:
//   warp 0      TMA: Q tile per piece, K tiles into a 4-stage ring.
//   warp 2      TMA: V tiles into a 6-stage ring (V is held longer than K);
//               the whole warp also allocates and frees TMEM.
//   warp 1      tcgen05 issuer for S = Q K^T into TMEM buffer S_w.
//   warp 3      tcgen05 issuer for O_w += P V (V read MN-major).
//   warps 4-11  two softmax warpgroups taking alternate tiles, one thread per
//               row: S from TMEM, mask, online softmax in the exp2 domain
//               (rescaling O in TMEM only when the running max grows by more
//               than 2^8, exact because the final normaliser uses the same
//               reference), P as bf16 into swizzled shared memory.  At the end
//               of a piece group 0 merges both groups' (m, l, O) and writes the
//               piece's partial result.
// A second, small kernel merges the partials of each segment by log-sum-exp
// and writes bf16 output.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "host.h"

namespace orthrus {
namespace attn {

constexpr int TN = 64;        // keys per tile
constexpr int NK = 4;         // K ring stages (a K tile is released once S = Q K^T is done)
constexpr int NV = 6;         // V ring stages (a V tile is held until O += P V is done)
constexpr int ROWS = 128;     // query rows per tile (tcgen05 M)
constexpr int THREADS = 384;  // 12 warps: TMA, MMA, TMEM alloc, spare, 2 softmax groups
constexpr int TMEM_COLS = 512;
constexpr int TMEM_O = 128;   // O accumulators at 128 and 256 (S buffers at 0 and TN)

template <int D>
struct Layout {
  static constexpr int CHUNKS = D / 64;            // 128-byte column chunks of a row
  static constexpr int Q_CHUNK = ROWS * 128;
  static constexpr int KV_CHUNK = TN * 128;
  static constexpr int Q_BYTES = CHUNKS * Q_CHUNK;
  static constexpr int KV_BYTES = CHUNKS * KV_CHUNK;
  static constexpr int P_BYTES = ROWS * TN * 2;     // one 128-byte chunk per row
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NV * KV_BYTES;
  static constexpr int OFF_ML = OFF_P + 2 * P_BYTES;   // [ROWS] float2 handed WG1 -> WG0
  static constexpr int OFF_BAR = OFF_ML + ROWS * 8;
  static constexpr int NBAR = 2 * NK + 2 * NV + 13;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;        // room to align the base to 1024
};

struct Params {
  const int32_t* ctx_lens;
  float* part_o;      // [slots][ROWS][D] unnormalised O of each piece
  float2* part_ml;    // [slots][ROWS] (m in log2 units, l)
  int32_t* dev_status;
  int B, K, Hq, Hkv, G, Gc, nhc, cap, mask_mode;
  float sl2;          // softmax scale * log2(e)
};

__device__ __forceinline__ int clamp_len(int L, const Params& p) {
  return L < 0 ? 0 : (L > p.cap - p.K ? p.cap - p.K : L);
}
__device__ __forceinline__ int n_tiles(int L, const Params& p) { return (L + p.K + TN - 1) / TN; }

// Walks the flattened tile space: sequences b, then segments (KV head g,
// head chunk hc) of b, then 64-key tiles t of the segment.
struct Cursor {
  long long base;  // first tile of sequence b
  int b, L, nt, seg, t;
};

__device__ __forceinline__ void cursor_load(Cursor& c, const Params& p) {
  c.L = clamp_len(__ldg(p.ctx_lens + c.b), p);
  c.nt = n_tiles(c.L, p);
}

__device__ void cursor_seek(Cursor& c, const Params& p, long long x) {
  const int nseg = p.Hkv * p.nhc;
  c.b = 0;
  c.base = 0;
  cursor_load(c, p);
  while (c.b + 1 < p.B && x >= c.base + static_cast<long long>(nseg) * c.nt) {
    c.base += static_cast<long long>(nseg) * c.nt;
    ++c.b;
    cursor_load(c, p);
  }
  const long long local = x - c.base;
  c.seg = static_cast<int>(local / c.nt);
  c.t = static_cast<int>(local % c.nt);
}

__device__ __forceinline__ void cursor_next(Cursor& c, const Params& p) {
  if (++c.t < c.nt) return;
  c.t = 0;
  const int nseg = p.Hkv * p.nhc;
  if (++c.seg < nseg) return;
  c.seg = 0;
  c.base += static_cast<long long>(nseg) * c.nt;
  if (++c.b < p.B) cursor_load(c, p);
}

__device__ long long total_tiles(const Params& p, bool report_errors) {
  long long T = 0;
  const int nseg = p.Hkv * p.nhc;
  for (int b = 0; b < p.B; ++b) {
    const int raw = __ldg(p.ctx_lens + b);
    if (report_errors && (raw < 0 || raw > p.cap - p.K)) report(p.dev_status, ORTHRUS_ECAPACITY);
    T += static_cast<long long>(nseg) * n_tiles(clamp_len(raw, p), p);
  }
  return T;
}

// First tile of CTA c when T tiles are split over P CTAs.
__device__ __forceinline__ long long cta_start(long long c, long long T, long long P) {
  return c * T / P;
}
// The CTA whose range contains tile x (the last c with cta_start(c) <= x).
__device__ __forceinline__ long long cta_of(long long x, long long T, long long P) {
  return ((x + 1) * P - 1) / T;
}

// Wait that ignores the abort flag, used only to drain in-flight async work
// before the CTA exits.
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity, int32_t* status) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) {  // 200 ms
      report(status, ORTHRUS_ETIMEOUT);
      return;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
    attn_splitkv_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const Params p) {
  using Ly = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sb0 = raw_addr + pad;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t bar = sb0 + Ly::OFF_BAR;
  auto full_k = [&](int s) { return bar + 8u * s; };
  auto empty_k = [&](int s) { return bar + 8u * (NK + s); };
  auto full_v = [&](int s) { return bar + 8u * (2 * NK + s); };
  auto empty_v = [&](int s) { return bar + 8u * (2 * NK + NV + s); };
  const uint32_t bar2 = bar + 8u * (2 * NK + 2 * NV);
  const uint32_t q_full = bar2;
  const uint32_t q_empty = bar2 + 8u;
  auto s_full = [&](int i) { return bar2 + 8u * (2 + i); };
  auto s_free = [&](int i) { return bar2 + 8u * (4 + i); };
  auto p_full = [&](int i) { return bar2 + 8u * (6 + i); };
  auto p_empty = [&](int i) { return bar2 + 8u * (8 + i); };
  const uint32_t o_full = bar2 + 8u * 10;
  const uint32_t o_free = bar2 + 8u * 11;
  const uint32_t mma_done = bar2 + 8u * 12;  // both MMA issuers commit once at exit
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly::OFF_MISC + 4);
  float2* ml_xchg = reinterpret_cast<float2*>(smem + Ly::OFF_ML);

  const long long T = total_tiles(p, blockIdx.x == 0 && threadIdx.x == 0);
  const long long Pc = gridDim.x;
  const long long x0 = cta_start(blockIdx.x, T, Pc);
  const long long x1 = cta_start(blockIdx.x + 1, T, Pc);
  const int n = static_cast<int>(x1 - x0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NK; ++s) {
      mbar_init(full_k(s), 1);
      mbar_init(empty_k(s), 1);
    }
    for (int s = 0; s < NV; ++s) {
      mbar_init(full_v(s), 1);
      mbar_init(empty_v(s), 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_free(i), 4);
      mbar_init(p_full(i), 4);
      mbar_init(p_empty(i), 1);
    }
    mbar_init(o_full, 1);
    mbar_init(o_free, 4);
    mbar_init(mma_done, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nseg = p.Hkv * p.nhc;

#define WAIT_OR(barrier, parity, on_fail) \
  if (!mbar_wait_bounded((barrier), (parity), abort_flag, p.dev_status)) on_fail
#define WARP_WAIT_OR(barrier, parity, on_fail) \
  if (!mbar_wait_warp((barrier), (parity), abort_flag, p.dev_status)) on_fail

  if (n > 0 && warp == 0 && lane == 0) {
    // ------------------------------------------------- Q and K producer
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    const uint64_t policy = policy_evict_first();
    Cursor cur;
    cursor_seek(cur, p, x0);
    int pieces = 0, issued = 0;
    const uint32_t q_tx = static_cast<uint32_t>(p.Gc * p.K * D * 2);
    for (int j = 0; j < n; ++j) {
      const bool first = (j == 0) || cur.t == 0;
      const int g = cur.seg / p.nhc, hc = cur.seg % p.nhc;
      if (first) {
        WAIT_OR(q_empty, (pieces & 1) ^ 1, break);
        mbar_arrive_expect_tx(q_full, q_tx);
        for (int c = 0; c < Ly::CHUNKS; ++c)
          tma_load_3d(sb0 + Ly::OFF_Q + c * Ly::Q_CHUNK, &tmQ, q_full, c * 64,
                      g * p.G + hc * p.Gc, cur.b * p.K);
        ++pieces;
      }
      const int stage = j % NK;
      const int row0 = (cur.b * p.Hkv + g) * p.cap + cur.t * TN;
      WAIT_OR(empty_k(stage), ((j / NK) & 1) ^ 1, break);
      mbar_arrive_expect_tx(full_k(stage), Ly::KV_BYTES);
      for (int c = 0; c < Ly::CHUNKS; ++c)
        tma_load_2d_hint(sb0 + Ly::OFF_K + stage * Ly::KV_BYTES + c * Ly::KV_CHUNK, &tmK,
                         full_k(stage), c * 64, row0, policy);
      ++issued;
      cursor_next(cur, p);
    }
    // Drain: every issued copy must have landed before the CTA may exit.
    for (int j = (issued > NK ? issued - NK : 0); j < issued; ++j)
      mbar_wait_drain(full_k(j % NK), (j / NK) & 1, p.dev_status);
    if (pieces > 0) mbar_wait_drain(q_full, (pieces - 1) & 1, p.dev_status);
  } else if (n > 0 && warp == 2 && lane == 0) {
    // ------------------------------------------------------- V producer
    prefetch_tmap(&tmV);
    const uint64_t policy = policy_evict_first();
    Cursor cur;
    cursor_seek(cur, p, x0);
    int issued = 0;
    for (int j = 0; j < n; ++j) {
      const int g = cur.seg / p.nhc;
      const int stage = j % NV;
      const int row0 = (cur.b * p.Hkv + g) * p.cap + cur.t * TN;
      WAIT_OR(empty_v(stage), ((j / NV) & 1) ^ 1, break);
      mbar_arrive_expect_tx(full_v(stage), Ly::KV_BYTES);
      for (int c = 0; c < Ly::CHUNKS; ++c)
        tma_load_2d_hint(sb0 + Ly::OFF_V + stage * Ly::KV_BYTES + c * Ly::KV_CHUNK, &tmV,
                         full_v(stage), c * 64, row0, policy);
      ++issued;
      cursor_next(cur, p);
    }
    for (int j = (issued > NV ? issued - NV : 0); j < issued; ++j)
      mbar_wait_drain(full_v(j % NV), (j / NV) & 1, p.dev_status);
  } else if (n > 0 && warp == 1 && lane == 0) {
    // ------------------------------------------------ S = Q K^T issuer
    // Tile j belongs to softmax warpgroup w = j & 1 and lands in TMEM S_w.
    const uint32_t id_s = make_idesc_bf16_f32(ROWS, TN, false, false);
    Cursor cs;
    cursor_seek(cs, p, x0);
    int q_seen = 0;
    for (int j = 0; j < n; ++j) {
      const bool first = (j == 0) || cs.t == 0;
      const bool last = (j == n - 1) || cs.t == cs.nt - 1;
      if (first) {
        WAIT_OR(q_full, q_seen & 1, break);
        ++q_seen;
      }
      const int stage = j % NK;
      WAIT_OR(full_k(stage), (j / NK) & 1, break);
      const int w = j & 1;
      const int u = j >> 1;
      if (u >= 1) {
        WAIT_OR(s_free(w), (u - 1) & 1, break);
      }
      tc_fence_after();
      const uint32_t qa = sb0 + Ly::OFF_Q;
      const uint32_t ka = sb0 + Ly::OFF_K + stage * Ly::KV_BYTES;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t ad = make_sdesc(qa + (kk >> 2) * Ly::Q_CHUNK + (kk & 3) * 32, 16, 1024,
                                       kSwizzle128B);
        const uint64_t bd = make_sdesc(ka + (kk >> 2) * Ly::KV_CHUNK + (kk & 3) * 32, 16, 1024,
                                       kSwizzle128B);
        mma_bf16_ss(tmem + w * TN, ad, bd, id_s, kk > 0 ? 1u : 0u);
      }
      mma_commit(empty_k(stage));
      mma_commit(s_full(w));
      if (last) mma_commit(q_empty);
      cursor_next(cs, p);
    }
    // every MMA of both issuers must be complete before TMEM is released
    mma_commit(mma_done);
    mbar_wait_drain(mma_done, 0, p.dev_status);
  } else if (n > 0 && warp == 3 && lane == 0) {
    // ------------------------------------------------ O_w += P V issuer
    const uint32_t id_pv = make_idesc_bf16_f32(ROWS, D, false, true);
    Cursor cp;
    cursor_seek(cp, p, x0);
    int pieces_done = 0, jp = 0;
    for (int j = 0; j < n; ++j) {
      const bool first = (j == 0) || cp.t == 0;
      const bool last = (j == n - 1) || cp.t == cp.nt - 1;
      if (first) {
        jp = j;
        if (pieces_done > 0) {
          WAIT_OR(o_free, (pieces_done - 1) & 1, break);
        }
      }
      const int w = j & 1;
      WAIT_OR(p_full(w), (j >> 1) & 1, break);
      const int stage = j % NV;
      WAIT_OR(full_v(stage), (j / NV) & 1, break);
      tc_fence_after();
      const uint32_t pa = sb0 + Ly::OFF_P + w * Ly::P_BYTES;
      const uint32_t va = sb0 + Ly::OFF_V + stage * Ly::KV_BYTES;
      const bool fresh = (j - jp) < 2;  // first tile of group w in this piece
#pragma unroll
      for (int kk = 0; kk < TN / 16; ++kk) {
        const uint64_t ad = make_sdesc(pa + kk * 32, 16, 1024, kSwizzle128B);
        // V is [keys x d] with d contiguous: MN-major B operand.  16 keys per
        // step = two 8-row swizzle atoms (2048 B); d chunks Ly::KV_CHUNK apart.
        const uint64_t bd = make_sdesc(va + kk * 2048, Ly::KV_CHUNK, 1024, kSwizzle128B);
        mma_bf16_ss(tmem + TMEM_O + w * 128, ad, bd, id_pv, (fresh && kk == 0) ? 0u : 1u);
      }
      mma_commit(empty_v(stage));
      mma_commit(p_empty(w));
      if (last) {
        mma_commit(o_full);
        ++pieces_done;
      }
      cursor_next(cp, p);
    }
    mma_commit(mma_done);
    mbar_wait_drain(mma_done, 0, p.dev_status);
  } else if (n > 0 && warp >= 4) {
    // ------------------------------------------------ softmax + epilogue
    const int w = (warp - 4) >> 2;            // softmax warpgroup: even / odd tiles
    const int r = (warp & 3) * 32 + lane;     // query row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t t_s = lane_base + w * TN;
    const uint32_t t_o = lane_base + TMEM_O + w * 128;
    const int rows_valid = p.Gc * p.K;
    const int i_row = r / p.Gc;
    const float sl2 = p.sl2;
    Cursor cur;
    cursor_seek(cur, p, x0);
    int pieces = 0, jp = 0;
    float m_used = -INFINITY, l_sum = 0.f;
    for (int j = 0; j < n; ++j) {
      const bool first = (j == 0) || cur.t == 0;
      const bool last = (j == n - 1) || cur.t == cur.nt - 1;
      if (first) {
        jp = j;
        m_used = -INFINITY;
        l_sum = 0.f;
      }
      if ((j & 1) == w) {
        const bool fresh = (j - jp) < 2;
        const int u = j >> 1;
        const int kv_end = cur.L + p.K;
        const int lim = (r >= rows_valid) ? 0
                        : (p.mask_mode == ORTHRUS_MASK_DIFF ? kv_end : cur.L + i_row + 1);
        const int tile0 = cur.t * TN;
        WARP_WAIT_OR(s_full(w), u & 1, break);
        tc_fence_after();
        uint32_t sr[TN];
        tmem_ld64(t_s, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free(w));

        if (tile0 + TN > cur.L + 1) {
          // Tail tile: some keys lie past some row's limit.  Interior tiles
          // (every key < L + 1) skip this entirely.
          const int lim = (r >= rows_valid) ? 0
                          : (p.mask_mode == ORTHRUS_MASK_DIFF ? kv_end : cur.L + i_row + 1);
#pragma unroll
          for (int c = 0; c < TN; ++c)
            if (tile0 + c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < TN; c += 8) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            mx4[q] = fmax3(mx4[q], __uint_as_float(sr[c + 2 * q]),
                           __uint_as_float(sr[c + 2 * q + 1]));
        }
        const float mx = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]) * sl2;
        bool waited = false;
        float m_new = m_used;
        if (fresh) {
          m_new = mx;
        } else if (__any_sync(0xFFFFFFFFu, mx > m_used + 8.f)) {
          m_new = fmaxf(m_used, mx);
          const float f = (m_new == -INFINITY) ? 1.f
                          : (m_used == -INFINITY ? 0.f : fast_exp2(m_used - m_new));
          // O_w may only be touched once this group's previous P*V completed.
          WARP_WAIT_OR(p_empty(w), (u - 1) & 1, break);
          waited = true;
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(t_o + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
            tmem_st32(t_o + c0, o);
          }
          tmem_wait_st();
          l_sum *= f;
        }
        m_used = m_new;
        const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
        // p = 2^(s*sl2 - m): scale and shift as packed f32x2 FMAs, exp2 on the
        // SFU, row sum as packed adds in four independent chains.
        const float2 sc2 = make_float2(sl2, sl2);
        const float2 nm2 = make_float2(-m_eff, -m_eff);
        float2 acc2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
        float x[TN];
#pragma unroll
        for (int c = 0; c < TN; c += 2) {
          const float2 a2 = __ffma2_rn(
              make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nm2);
          const float2 e2 = make_float2(fast_exp2(a2.x), fast_exp2(a2.y));
          x[c] = e2.x;
          x[c + 1] = e2.y;
          acc2[(c >> 1) & 3] = __fadd2_rn(acc2[(c >> 1) & 3], e2);
        }
        const float2 t2 = __fadd2_rn(__fadd2_rn(acc2[0], acc2[1]), __fadd2_rn(acc2[2], acc2[3]));
        l_sum += t2.x + t2.y;

        if (tile0 + TN > kv_end) {
          // The tile runs past the valid keys: zero those V rows so that stale
          // or NaN cache contents cannot reach O through 0 * NaN.
          const int stage = j % NV;
          WARP_WAIT_OR(full_v(stage), (j / NV) & 1, break);
          const int nv = kv_end - tile0 > 0 ? kv_end - tile0 : 0;
          const int per_chunk = (TN - nv) * 8;
          uint8_t* vt = smem + Ly::OFF_V + stage * Ly::KV_BYTES;
          for (int q = r; q < per_chunk * Ly::CHUNKS; q += ROWS) {
            const int ch = q / per_chunk, rem = q % per_chunk;
            *reinterpret_cast<uint4*>(vt + ch * Ly::KV_CHUNK + (nv + rem / 8) * 128 +
                                      (rem % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        if (u >= 1 && !waited) {
          WARP_WAIT_OR(p_empty(w), (u - 1) & 1, break);
        }
        uint8_t* prow = smem + Ly::OFF_P + w * Ly::P_BYTES + r * 128;
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {
          uint4 v;
          v.x = pack_bf16x2(x[8 * pc + 0], x[8 * pc + 1]);
          v.y = pack_bf16x2(x[8 * pc + 2], x[8 * pc + 3]);
          v.z = pack_bf16x2(x[8 * pc + 4], x[8 * pc + 5]);
          v.w = pack_bf16x2(x[8 * pc + 6], x[8 * pc + 7]);
          *reinterpret_cast<uint4*>(prow + ((pc ^ (r & 7)) * 16)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(w));
      }

      if (last) {
        // Piece epilogue: merge the two groups' (m, l, O) and publish it.
        WARP_WAIT_OR(o_full, pieces & 1, break);
        tc_fence_after();
        if (w == 1) ml_xchg[r] = make_float2(m_used, l_sum);
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (w == 0) {
          const float2 o1 = ml_xchg[r];
          const float M = fmaxf(m_used, o1.x);
          const float a0 = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - M);
          const float a1 = (o1.x == -INFINITY) ? 0.f : fast_exp2(o1.x - M);
          const long long slot = static_cast<long long>(cur.b) * nseg + cur.seg + blockIdx.x;
          float* dst = p.part_o + (slot * ROWS + r) * D;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o0[32], o1r[32];
            tmem_ld32(t_o + c0, o0);
            tmem_ld32(t_o + 128 + c0, o1r);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; k += 4) {
              float4 v;
              v.x = (a0 != 0.f ? a0 * __uint_as_float(o0[k]) : 0.f) +
                    (a1 != 0.f ? a1 * __uint_as_float(o1r[k]) : 0.f);
              v.y = (a0 != 0.f ? a0 * __uint_as_float(o0[k + 1]) : 0.f) +
                    (a1 != 0.f ? a1 * __uint_as_float(o1r[k + 1]) : 0.f);
              v.z = (a0 != 0.f ? a0 * __uint_as_float(o0[k + 2]) : 0.f) +
                    (a1 != 0.f ? a1 * __uint_as_float(o1r[k + 2]) : 0.f);
              v.w = (a0 != 0.f ? a0 * __uint_as_float(o0[k + 3]) : 0.f) +
                    (a1 != 0.f ? a1 * __uint_as_float(o1r[k + 3]) : 0.f);
              *reinterpret_cast<float4*>(dst + c0 + k) = v;
            }
          }
          p.part_ml[slot * ROWS + r] = make_float2(M, a0 * l_sum + a1 * o1.y);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free);
        }
        ++pieces;
      }
      cursor_next(cur, p);
    }
  }
#undef WAIT_OR
#undef WARP_WAIT_OR

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Merge the pieces of each (sequence, KV head, head chunk) segment by
// log-sum-exp.  One warp per query row; lane owns D/32 consecutive columns.
// The pieces' (m, l) pairs are read lane-parallel and their O rows are
// fetched with independent loads so the merge is bandwidth-, not
// latency-bound.
template <int D>
__global__ void __launch_bounds__(128) attn_combine_kernel(const Params p, int grid_ctas,
                                                           __nv_bfloat16* __restrict__ out) {
  constexpr int PER = D / 32;
  const int s = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * 4 + warp;
  const int nseg = p.Hkv * p.nhc;
  const int b = s / nseg, seg = s % nseg;
  const int g = seg / p.nhc, hc = seg % p.nhc;
  const int i = r / p.Gc, hh = r % p.Gc;
  if (i >= p.K || hc * p.Gc + hh >= p.G) return;

  long long T = 0, Ts = 0;
  int nt_b = 1;
  for (int bb = 0; bb < p.B; ++bb) {
    const int nt = n_tiles(clamp_len(__ldg(p.ctx_lens + bb), p), p);
    if (bb == b) {
      Ts = T + static_cast<long long>(seg) * nt;
      nt_b = nt;
    }
    T += static_cast<long long>(nseg) * nt;
  }
  const long long P = grid_ctas;
  const long long c0 = cta_of(Ts, T, P), c1 = cta_of(Ts + nt_b - 1, T, P);

  float M = -INFINITY;
  for (long long base = c0; base <= c1; base += 32) {
    const long long c = base + lane;
    if (c <= c1 && cta_start(c, T, P) != cta_start(c + 1, T, P))
      M = fmaxf(M, __ldcg(&p.part_ml[(s + c) * ROWS + r]).x);
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, m));

  float acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.f;
  float Lp = 0.f;
  for (long long base = c0; base <= c1; base += 32) {
    const long long c = base + lane;
    float wgt = 0.f;
    if (c <= c1 && cta_start(c, T, P) != cta_start(c + 1, T, P)) {
      const float2 ml = __ldcg(&p.part_ml[(s + c) * ROWS + r]);
      wgt = (ml.x == -INFINITY) ? 0.f : fast_exp2(ml.x - M);
      Lp += wgt * ml.y;
    }
    const int cnt = static_cast<int>(c1 - base + 1 < 32 ? c1 - base + 1 : 32);
    for (int k0 = 0; k0 < cnt; k0 += 8) {
      // eight independent loads in flight, then the weighted sums
      float wk[8];
      float v[8][PER];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        wk[k] = __shfl_sync(0xFFFFFFFFu, wgt, (k0 + k) & 31);
        const bool live = (k0 + k < cnt) && wk[k] != 0.f;
        const float* src = p.part_o + ((s + base + k0 + k) * ROWS + r) * D + lane * PER;
        if constexpr (PER == 4) {
          const float4 t = live ? __ldcg(reinterpret_cast<const float4*>(src))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
          v[k][0] = t.x;
          v[k][1] = t.y;
          v[k][2] = t.z;
          v[k][3] = t.w;
        } else {
          const float2 t = live ? __ldcg(reinterpret_cast<const float2*>(src))
                                : make_float2(0.f, 0.f);
          v[k][0] = t.x;
          v[k][1] = t.y;
        }
        if (!live) wk[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k)
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] += wk[k] * v[k][e];
    }
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) Lp += __shfl_xor_sync(0xFFFFFFFFu, Lp, m);
  const float inv = Lp > 0.f ? 1.f / Lp : 0.f;
  const int h = g * p.G + hc * p.Gc + hh;
  __nv_bfloat16* dst = out + ((static_cast<long long>(b) * p.K + i) * p.Hq + h) * D + lane * PER;
#pragma unroll
  for (int k = 0; k < PER; k += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + k) = __floats2bfloat162_rn(acc[k] * inv,
                                                                        acc[k + 1] * inv);
}

struct Shape {
  int B, K, Hq, Hkv, d, G, Gc, nhc, S;
};

int check_shape(int B, int Hq, int Hkv, int d, int K, Shape* sh) {
  if (K < 1 || K > 32) return ORTHRUS_EINVAL;
  if (B < 0 || Hq < 1 || Hkv < 1) return ORTHRUS_EINVAL;
  if (Hq % Hkv != 0) return ORTHRUS_ESHAPE;
  if (d != 64 && d != 128) return ORTHRUS_EUNSUPPORTED;
  sh->B = B;
  sh->K = K;
  sh->Hq = Hq;
  sh->Hkv = Hkv;
  sh->d = d;
  sh->G = Hq / Hkv;
  const int per = ROWS / K;  // heads per 128-row tile
  sh->Gc = sh->G < per ? sh->G : per;
  sh->nhc = (sh->G + sh->Gc - 1) / sh->Gc;
  sh->S = B * Hkv * sh->nhc;
  return ORTHRUS_OK;
}

size_t workspace_bytes(const Shape& sh, int sms) {
  const size_t slots = static_cast<size_t>(sh.S) + static_cast<size_t>(sms);
  const size_t o_bytes = slots * ROWS * sh.d * sizeof(float);
  const size_t ml_bytes = slots * ROWS * sizeof(float2);
  return o_bytes + ml_bytes + 256;
}

template <int D>
int launch(const Shape& sh, const void* q, const orthrus_kv_cache* cache, int mask_mode,
           void* out, void* ws, int sms, int32_t* dev_status, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(sh.Hq),
                              static_cast<uint64_t>(sh.B) * sh.K};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2,
                                 static_cast<uint64_t>(sh.Hq) * D * 2};
    const uint32_t box[3] = {64u, static_cast<uint32_t>(sh.Gc), static_cast<uint32_t>(sh.K)};
    const int rc = encode_tmap_bf16(&tq, q, 3, dims, strides, box);
    if (rc != ORTHRUS_OK) return rc;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(D),
                              static_cast<uint64_t>(sh.B) * sh.Hkv * cache->cap};
    const uint64_t strides[1] = {static_cast<uint64_t>(D) * 2};
    const uint32_t box[2] = {64u, static_cast<uint32_t>(TN)};
    int rc = encode_tmap_bf16(&tk, cache->k, 2, dims, strides, box);
    if (rc != ORTHRUS_OK) return rc;
    rc = encode_tmap_bf16(&tv, cache->v, 2, dims, strides, box);
    if (rc != ORTHRUS_OK) return rc;
  }
  Params p;
  p.ctx_lens = cache->ctx_lens;
  const size_t slots = static_cast<size_t>(sh.S) + static_cast<size_t>(sms);
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.part_o = reinterpret_cast<float*>(w);
  p.part_ml = reinterpret_cast<float2*>(w + slots * ROWS * D * sizeof(float));
  p.dev_status = dev_status;
  p.B = sh.B;
  p.K = sh.K;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.G = sh.G;
  p.Gc = sh.Gc;
  p.nhc = sh.nhc;
  p.cap = cache->cap;
  p.mask_mode = mask_mode;
  p.sl2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));

  auto* kfn = attn_splitkv_kernel<D>;
  if (!opt_in_smem(reinterpret_cast<const void*>(kfn), Layout<D>::ALLOC)) return ORTHRUS_ECUDA;
  kfn<<<sms, THREADS, Layout<D>::ALLOC, stream>>>(tq, tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return ORTHRUS_ECUDA;
  const dim3 cgrid(sh.S, (sh.Gc * sh.K + 3) / 4);
  attn_combine_kernel<D><<<cgrid, 128, 0, stream>>>(p, sms, static_cast<__nv_bfloat16*>(out));
  if (cudaGetLastError() != cudaSuccess) return ORTHRUS_ECUDA;
  return ORTHRUS_OK;
}

}  // namespace attn
}  // namespace orthrus

using namespace orthrus;

extern "C" int orthrus_block_attn_workspace_size(int B, int Hq, int Hkv, int d, int K,
                                                 size_t* bytes) {
  if (bytes == nullptr) return ORTHRUS_EINVAL;
  attn::Shape sh;
  int rc = attn::check_shape(B, Hq, Hkv, d, K, &sh);
  if (rc != ORTHRUS_OK) return rc;
  int sms = 0;
  rc = current_sm_count(&sms);
  if (rc != ORTHRUS_OK) return rc;
  *bytes = attn::workspace_bytes(sh, sms);
  return ORTHRUS_OK;
}

extern "C" int orthrus_block_attn(const void* q, const orthrus_kv_cache* cache, int Hq, int K,
                                  int mask_mode, void* out, void* workspace, size_t ws_bytes,
                                  int32_t* dev_status, void* stream) {
  if (q == nullptr || cache == nullptr || out == nullptr) return ORTHRUS_EINVAL;
  if (mask_mode != ORTHRUS_MASK_DIFF && mask_mode != ORTHRUS_MASK_AR) return ORTHRUS_EINVAL;
  attn::Shape sh;
  int rc = attn::check_shape(cache->B, Hq, cache->Hkv, cache->d, K, &sh);
  if (rc != ORTHRUS_OK) return rc;
  if (cache->k == nullptr || cache->v == nullptr || cache->ctx_lens == nullptr)
    return ORTHRUS_EINVAL;
  if (cache->cap < K) return ORTHRUS_ESHAPE;
  if (static_cast<long long>(cache->B) * cache->Hkv * cache->cap >= (1ll << 31) ||
      static_cast<long long>(cache->B) * K * Hq >= (1ll << 31))
    return ORTHRUS_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(cache->k) || !aligned16(cache->v) || !aligned16(out) ||
      !aligned16(workspace))
    return ORTHRUS_EALIGN;
  if (sh.B == 0) return ORTHRUS_OK;
  int sms = 0;
  rc = current_sm_count(&sms);
  if (rc != ORTHRUS_OK) return rc;
  if (workspace == nullptr || ws_bytes < attn::workspace_bytes(sh, sms))
    return ORTHRUS_EWORKSPACE;
  const cudaStream_t s = as_stream(stream);
  if (sh.d == 128) return attn::launch<128>(sh, q, cache, mask_mode, out, workspace, sms,
                                            dev_status, s);
  return attn::launch<64>(sh, q, cache, mask_mode, out, workspace, sms, dev_status, s);
}
