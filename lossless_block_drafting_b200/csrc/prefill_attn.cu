// Causal attention over a prompt chunk: the AR view's pre-filling pass.
//
// Method: gist.science summary of "Orthrus: Memory-Efficient Parallel Token
// Generation via Dual-View Diffusion", technical summary 2.1 item 1 (the frozen
// AR head's only job is to pre-fill the context into the shared KV cache that
// both views then read) and the paper's abstract (the autoregressive head
// executes context pre-filling).  Row i of sequence b sits at position
// L_b + i and attends keys [0, L_b + i + 1): the same mask as the AR view's
// block attention, with the chunk in place of the K-token block (L_b = 0 for a
// whole prompt, L_b > 0 for a later chunk of a long one).
//
// Design (B200, sm_100a).  Compute-bound (4 flop per key per query per head
// dimension, ~P^2/2 keys), so the work is cut into tiles of 128 consecutive
// positions of one query head (the tcgen05 M = 128 rows) and every CTA owns
// TWO such tiles -- two query heads of one GQA group at the same positions --
// that share each 128-key K/V group it loads: the shared-memory fill per MMA
// is halved.  One CTA per SM at a time (192 KB of shared memory, all 512 TMEM
// columns), the longest (latest) position tiles launched first.
//   warp 0      TMA: both Q tiles once, then K and V groups into 2-stage rings.
//   warp 1      the single tcgen05 issuer, in the order
//                 S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...
//               S_t and P_t share tile t's 128 TMEM columns (P overwrites the
//               first 64 as bf16), so S_t(j+1) is issued once PV_t(j) has
//               completed.  The two tiles settle half a period apart: the
//               tensor core works on one while the other's softmax runs.
//   warp 2      TMEM allocation.
//   warps 4-7   softmax of tile 0, warps 8-11 of tile 1: one thread per row,
//               64 keys at a time, exp2 against a running reference maximum
//               (O is rescaled only when a row's maximum grows by more than
//               2^8, exact because the final normaliser uses the same
//               reference), causal masking only on the groups that reach the
//               diagonal; finally O / l in bf16 to the output.
#include <cuda_bf16.h>

#include <cmath>

#include "common.cuh"
#include "host.h"

namespace orthrus {
namespace pre {

constexpr int ROWS = 128;     // positions per tile (tcgen05 M)
constexpr int KG = 128;       // keys per group
constexpr int HK = 64;        // keys per softmax half
constexpr int THREADS = 384;
constexpr int NST = 2;        // K and V ring stages

template <int D>
struct Layout {
  static constexpr int CHUNKS = D / 64;            // 128-byte column chunks of a row
  static constexpr int Q_CHUNK = ROWS * 128;       // one tile's chunk
  static constexpr int Q_TILE = CHUNKS * Q_CHUNK;
  static constexpr int KV_CHUNK = KG * 128;        // one group's chunk
  static constexpr int KV_BYTES = CHUNKS * KV_CHUNK;
  static constexpr int OFF_Q = 0;                  // [2 tiles]
  static constexpr int OFF_K = OFF_Q + 2 * Q_TILE;
  static constexpr int OFF_V = OFF_K + NST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NST * KV_BYTES;
  static constexpr int NBAR = 1 + 4 * NST + 2 * 3 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;       // room to align the base to 1024
  // TMEM columns: S/P of tile t at t * 128, O of tile t at 256 + t * D
  static constexpr int TMEM_O = 256;
};

struct Params {
  const int32_t* ctx_lens;
  __nv_bfloat16* out;  // [B, P, Hq, D]
  int32_t* dev_status;
  unsigned long long wait_ns;
  int B, P, Hq, Hkv, G, npairs, nqt, cap;
  float sl2;           // softmax scale * log2(e)
};

template <int D, bool kShortWait>
__global__ void __launch_bounds__(THREADS, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const Params p) {
  using Ly = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_addr & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t sb0 = raw_addr + pad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const uint32_t bar = sb0 + Ly::OFF_BAR;
  const uint32_t q_full = bar;
  auto k_full = [&](int s) { return bar + 8u * (1 + s); };
  auto k_empty = [&](int s) { return bar + 8u * (1 + NST + s); };
  auto v_full = [&](int s) { return bar + 8u * (1 + 2 * NST + s); };
  auto v_empty = [&](int s) { return bar + 8u * (1 + 3 * NST + s); };
  auto s_full = [&](int t) { return bar + 8u * (1 + 4 * NST + t); };       // S_t(j) in TMEM
  auto p_full = [&](int t) { return bar + 8u * (1 + 4 * NST + 2 + t); };   // P_t(j) written
  auto pv_done = [&](int t) { return bar + 8u * (1 + 4 * NST + 4 + t); };  // PV_t(j) complete
  const uint32_t mma_done = bar + 8u * (1 + 4 * NST + 6);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly::OFF_MISC + 4);

  // This CTA's unit: the latest position tiles first (they have the most keys).
  const int per_qt = p.B * p.Hkv * p.npairs;
  const int qt = p.nqt - 1 - static_cast<int>(blockIdx.x) / per_qt;
  const int rest = static_cast<int>(blockIdx.x) % per_qt;
  const int b = rest / (p.Hkv * p.npairs);
  const int g = (rest / p.npairs) % p.Hkv;
  const int hp = rest % p.npairs;
  const int h0 = g * p.G + 2 * hp;
  const bool two = 2 * hp + 1 < p.G;  // a second query head of the group exists
  const int p0 = qt * ROWS;

  grid_dep_launch();
  if (threadIdx.x == 32) {
    mbar_init(q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), 4);
      mbar_init(pv_done(t), 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  } else if (threadIdx.x == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  grid_dep_wait();  // ctx_lens, q and the cache may come from the previous kernel
  // Chunk start L and this CTA's key range [0, kend): the last valid row of the
  // tile attends keys up to L + min(p0 + 128, P) - 1.
  const int raw = __ldcg(p.ctx_lens + b);
  const int L = raw < 0 ? 0 : (raw > p.cap - p.P ? p.cap - p.P : raw);
  if (threadIdx.x == 0 && (raw < 0 || raw > p.cap - p.P) && qt == p.nqt - 1 && rest == 0)
    report(p.dev_status, ORTHRUS_ECAPACITY);
  const int rows_valid = p.P - p0 < ROWS ? p.P - p0 : ROWS;
  const int kend = L + p0 + rows_valid;
  const int ngroups = (kend + KG - 1) / KG;
  const int kvbase = (b * p.Hkv + g) * p.cap;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

#define WAIT_OR(barrier, parity, on_fail) \
  if (!mbar_wait_bounded<kShortWait>((barrier), (parity), abort_flag, p.dev_status, p.wait_ns)) on_fail
#define WARP_WAIT_OR(barrier, parity, on_fail) \
  if (!mbar_wait_warp<kShortWait>((barrier), (parity), abort_flag, p.dev_status, p.wait_ns)) on_fail

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    // K/V are re-read by the CTAs of later tiles: default L2 policy.
    mbar_arrive_expect_tx(q_full, static_cast<uint32_t>((two ? 2 : 1) * Ly::Q_TILE));
    for (int t = 0; t < (two ? 2 : 1); ++t)
      for (int c = 0; c < Ly::CHUNKS; ++c)
        tma_load_3d(sb0 + Ly::OFF_Q + t * Ly::Q_TILE + c * Ly::Q_CHUNK, &tmQ, q_full, c * 64,
                    h0 + t, b * p.P + p0);
    int nk = 0, nv = 0;  // K and V groups issued
    for (int j = 0; j < ngroups; ++j) {
      const int s = j % NST;
      WAIT_OR(k_empty(s), ((j / NST) & 1) ^ 1, break);
      mbar_arrive_expect_tx(k_full(s), Ly::KV_BYTES);
      for (int c = 0; c < Ly::CHUNKS; ++c)
        tma_load_2d(sb0 + Ly::OFF_K + s * Ly::KV_BYTES + c * Ly::KV_CHUNK, &tmK, k_full(s),
                    c * 64, kvbase + j * KG);
      ++nk;
      WAIT_OR(v_empty(s), ((j / NST) & 1) ^ 1, break);
      mbar_arrive_expect_tx(v_full(s), Ly::KV_BYTES);
      for (int c = 0; c < Ly::CHUNKS; ++c)
        tma_load_2d(sb0 + Ly::OFF_V + s * Ly::KV_BYTES + c * Ly::KV_CHUNK, &tmV, v_full(s),
                    c * 64, kvbase + j * KG);
      ++nv;
    }
    // Drain: every copy issued must land before the CTA may exit (only the
    // last NST of each ring can still be in flight).
    for (int j = nk - NST < 0 ? 0 : nk - NST; j < nk; ++j)
      mbar_drain(k_full(j % NST), (j / NST) & 1, p.dev_status);
    for (int j = nv - NST < 0 ? 0 : nv - NST; j < nv; ++j)
      mbar_drain(v_full(j % NST), (j / NST) & 1, p.dev_status);
    mbar_drain(q_full, 0, p.dev_status);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    const uint32_t id_s = make_idesc_bf16_f32(ROWS, KG, false, false);
    const uint32_t id_pv = make_idesc_bf16_f32(ROWS, D, false, true);
    uint64_t qd[D / 16], kd[D / 16], vd[KG / 16];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      qd[kk] = make_sdesc(sb0 + Ly::OFF_Q + (kk >> 2) * Ly::Q_CHUNK + (kk & 3) * 32, 16, 1024,
                          kSwizzle128B);
      kd[kk] = make_sdesc(sb0 + Ly::OFF_K + (kk >> 2) * Ly::KV_CHUNK + (kk & 3) * 32, 16, 1024,
                          kSwizzle128B);
    }
#pragma unroll
    for (int kk = 0; kk < KG / 16; ++kk)
      // V is [keys x d], d contiguous: MN-major B operand; 16 keys per step are
      // two 8-row swizzle atoms (2048 B), d chunks Ly::KV_CHUNK apart.
      vd[kk] = make_sdesc(sb0 + Ly::OFF_V + kk * 2048, Ly::KV_CHUNK, 1024, kSwizzle128B);
    const uint64_t qtile = static_cast<uint64_t>(Ly::Q_TILE >> 4);
    const int nt = two ? 2 : 1;
    auto issue_s = [&](int t, int j) {
      const int s = j % NST;
      const uint64_t koff = static_cast<uint64_t>((s * Ly::KV_BYTES) >> 4);
      const uint32_t dst = tmem + t * KG;
      mma_bf16_ss(dst, qd[0] + t * qtile, kd[0] + koff, id_s, 0u);
#pragma unroll
      for (int kk = 1; kk < D / 16; ++kk)
        mma_bf16_ss(dst, qd[kk] + t * qtile, kd[kk] + koff, id_s, 1u);
      mma_commit(s_full(t));
    };
    auto issue_pv = [&](int t, int j) {
      const int s = j % NST;
      const uint64_t voff = static_cast<uint64_t>((s * Ly::KV_BYTES) >> 4);
      const uint32_t a_p = tmem + t * KG;  // P: 16 keys = 8 columns per step
      const uint32_t dst = tmem + Ly::TMEM_O + t * D;
      mma_bf16_ts(dst, a_p, vd[0] + voff, id_pv, j > 0 ? 1u : 0u);
#pragma unroll
      for (int kk = 1; kk < KG / 16; ++kk)
        mma_bf16_ts(dst, a_p + kk * 8, vd[kk] + voff, id_pv, 1u);
      mma_commit(pv_done(t));
    };
    bool ok = true;
    do {
      WAIT_OR(q_full, 0, { ok = false; break; });
      WAIT_OR(k_full(0), 0, { ok = false; break; });
      tc_fence_after();
      for (int t = 0; t < nt; ++t) issue_s(t, 0);
      mma_commit(k_empty(0));
      for (int j = 0; ok && j < ngroups; ++j) {
        const int s = j % NST;
        const bool more = j + 1 < ngroups;
        WAIT_OR(v_full(s), (j / NST) & 1, { ok = false; break; });
        for (int t = 0; t < nt; ++t) {
          // tile t: P_t(j) -> PV_t(j); once it has consumed P_t(j), S_t(j + 1)
          // may overwrite it.  The other tile's softmax runs meanwhile, so
          // the two tiles settle half a period apart.
          WAIT_OR(p_full(t), j & 1, { ok = false; break; });
          tc_fence_after();
          issue_pv(t, j);
          if (t == nt - 1) mma_commit(v_empty(s));
          if (more) {
            if (t == 0) {
              WAIT_OR(k_full((j + 1) % NST), ((j + 1) / NST) & 1, { ok = false; break; });
            }
            WAIT_OR(pv_done(t), j & 1, { ok = false; break; });
            tc_fence_after();
            issue_s(t, j + 1);
            if (t == nt - 1) mma_commit(k_empty((j + 1) % NST));
          }
        }
      }
    } while (0);
    (void)ok;
    mma_commit(mma_done);
    mbar_drain(mma_done, 0, p.dev_status);
  } else if (warp >= 4) {
    // ------------------------------------------------ softmax + epilogue
    const int t = (warp - 4) >> 2;          // the tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;   // row == TMEM lane == position offset
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t t_s = lane_base + t * KG;
    const uint32_t t_o = lane_base + Ly::TMEM_O + t * D;
    const bool active = t == 0 || two;
    const int lim = L + p0 + (r < rows_valid ? r : rows_valid - 1) + 1;  // keys < lim
    const int lim_min = L + p0 + 1;                                     // smallest row limit
    const float sl2 = p.sl2;
    const float2 sc2 = make_float2(sl2, sl2);
    float m_used = -INFINITY, l_sum = 0.f;
    bool fail = false;
    // V rows of a group past the CTA's last key (kend) are zeroed by the two
    // warpgroups together so stale or NaN cache contents never reach O.
    for (int j = 0; active && j < ngroups; ++j) {
      WARP_WAIT_OR(s_full(t), j & 1, { fail = true; break; });
      tc_fence_after();
      const int k0 = j * KG;
      if (k0 + KG > kend) {
        const int s = j % NST;
        WARP_WAIT_OR(v_full(s), (j / NST) & 1, { fail = true; break; });
        const int nv = kend - k0;
        const int per_chunk = (KG - nv) * 8;
        uint8_t* vt = smem + Ly::OFF_V + s * Ly::KV_BYTES;
        const int tid = threadIdx.x - 128 * (1 + t);
        if (t == 0 || !two) {
          for (int q = tid; q < per_chunk * Ly::CHUNKS; q += 128) {
            const int ch = q / per_chunk, rem = q % per_chunk;
            *reinterpret_cast<uint4*>(vt + ch * Ly::KV_CHUNK + (nv + rem / 8) * 128 +
                                      (rem % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
      }
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int kh = k0 + h * HK;
        float x[HK];
        float2 acc2[4];
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
          uint32_t sr[HK];
          tmem_ld64(t_s + h * HK, sr);
          tmem_wait_ld();
          if (kh + HK > lim_min) {
#pragma unroll
            for (int c = 0; c < HK; ++c)
              if (kh + c >= lim) sr[c] = __float_as_uint(-INFINITY);
          }
          const bool take_max = (j == 0 && h == 0) || pass == 1;
          if (take_max) {
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < HK; c += 8) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                mx4[q] = fmax3(mx4[q], __uint_as_float(sr[c + 2 * q]),
                               __uint_as_float(sr[c + 2 * q + 1]));
            }
            const float mx = fmax3(fmaxf(mx4[0], mx4[1]), mx4[2], mx4[3]) * sl2;
            if (pass == 0) {
              m_used = mx;
            } else {
              const float m_new = fmaxf(m_used, mx);
              const float f = (m_new == -INFINITY) ? 1.f
                              : (m_used == -INFINITY ? 0.f : fast_exp2(m_used - m_new));
              if (j > 0) {
                // O_t holds PV_t up to group j - 1: wait for the last one.
                WARP_WAIT_OR(pv_done(t), (j - 1) & 1, { fail = true; break; });
                tc_fence_after();
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 16) {
                  uint32_t o[16];
                  tmem_ld16(t_o + c0, o);
                  tmem_wait_ld();
#pragma unroll
                  for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
                  tmem_st16(t_o + c0, o);
                }
                tmem_wait_st();
              }
              // the first half's P of this group (already in TMEM) was built
              // against the old reference: scale it too
              if (h == 1) {
                uint32_t pk0[HK / 2];
                tmem_ld32(t_s, pk0);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < HK / 2; ++c) {
                  const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162*>(&pk0[c]);
                  pk0[c] = pack_bf16x2(__low2float(v2) * f, __high2float(v2) * f);
                }
                tmem_st32(t_s, pk0);
                tmem_wait_st();
              }
              l_sum *= f;
              m_used = m_new;
            }
          }
          const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
          const float2 nm2 = make_float2(-m_eff, -m_eff);
#pragma unroll
          for (int q = 0; q < 4; ++q) acc2[q] = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < HK; c += 2) {
            const float2 a2 = __ffma2_rn(
                make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nm2);
            const float2 e2 = make_float2(fast_exp2(a2.x), fast_exp2(a2.y));
            x[c] = e2.x;
            x[c + 1] = e2.y;
            acc2[(c >> 1) & 3] = __fadd2_rn(acc2[(c >> 1) & 3], e2);
          }
          if (take_max) break;
          const float2 ts2 = __fadd2_rn(__fadd2_rn(acc2[0], acc2[1]), __fadd2_rn(acc2[2], acc2[3]));
          if (!__any_sync(0xFFFFFFFFu, !(ts2.x + ts2.y <= 256.f))) break;
        }
        if (fail) break;
        const float2 t2 = __fadd2_rn(__fadd2_rn(acc2[0], acc2[1]), __fadd2_rn(acc2[2], acc2[3]));
        l_sum += t2.x + t2.y;
        // P of this half (64 keys = 32 columns) over dead S columns: half 0
        // to [0, 32) of S_t, half 1 to [32, 64) (half 0's S, consumed)
        uint32_t pk[HK / 2];
#pragma unroll
        for (int c = 0; c < HK / 2; ++c) pk[c] = pack_bf16x2(x[2 * c], x[2 * c + 1]);
        tmem_st32(t_s + h * (HK / 2), pk);
        tmem_wait_st();
      }
      if (fail) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full(t));
    }
    if (active && !fail) {
      // Epilogue: O_t / l in bf16, once the last PV_t is complete.  The TMEM
      // loads are warp-collective: every lane takes part, and only the rows
      // inside the chunk are stored.
      WARP_WAIT_OR(pv_done(t), (ngroups - 1) & 1, fail = true);
      if (!fail) {
        tc_fence_after();
        const bool store = r < rows_valid;
        const float inv = l_sum > 0.f ? 1.f / l_sum : 0.f;
        __nv_bfloat16* dst =
            p.out + ((static_cast<long long>(b) * p.P + p0 + (store ? r : 0)) * p.Hq + h0 + t) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(t_o + c0, o);
          tmem_wait_ld();
          if (store) {
#pragma unroll
            for (int k = 0; k < 32; k += 8) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[k]) * inv, __uint_as_float(o[k + 1]) * inv);
              v.y = pack_bf16x2(__uint_as_float(o[k + 2]) * inv, __uint_as_float(o[k + 3]) * inv);
              v.z = pack_bf16x2(__uint_as_float(o[k + 4]) * inv, __uint_as_float(o[k + 5]) * inv);
              v.w = pack_bf16x2(__uint_as_float(o[k + 6]) * inv, __uint_as_float(o[k + 7]) * inv);
              *reinterpret_cast<uint4*>(dst + c0 + k) = v;
            }
          }
        }
      }
    }
  }
#undef WAIT_OR
#undef WARP_WAIT_OR

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
int launch(const void* q, const orthrus_kv_cache* cache, int Hq, int P, void* out,
           int32_t* dev_status, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(Hq),
                              static_cast<uint64_t>(cache->B) * P};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(Hq) * D * 2};
    const uint32_t box[3] = {64u, 1u, static_cast<uint32_t>(ROWS)};
    const int rc = encode_tmap_bf16(&tq, q, 3, dims, strides, box);
    if (rc != ORTHRUS_OK) return rc;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(D),
                              static_cast<uint64_t>(cache->B) * cache->Hkv * cache->cap};
    const uint64_t strides[1] = {static_cast<uint64_t>(D) * 2};
    const uint32_t box[2] = {64u, static_cast<uint32_t>(KG)};
    int rc = encode_tmap_bf16(&tk, cache->k, 2, dims, strides, box);
    if (rc == ORTHRUS_OK) rc = encode_tmap_bf16(&tv, cache->v, 2, dims, strides, box);
    if (rc != ORTHRUS_OK) return rc;
  }
  Params p;
  p.ctx_lens = cache->ctx_lens;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.dev_status = dev_status;
  p.wait_ns = wait_limit_ns();
  p.B = cache->B;
  p.P = P;
  p.Hq = Hq;
  p.Hkv = cache->Hkv;
  p.G = Hq / cache->Hkv;
  p.npairs = (p.G + 1) / 2;
  p.nqt = (P + ROWS - 1) / ROWS;
  p.cap = cache->cap;
  p.sl2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  const long long units = static_cast<long long>(p.B) * p.Hkv * p.npairs * p.nqt;
  if (units >= (1ll << 31)) return ORTHRUS_EUNSUPPORTED;
  auto* kfn = p.wait_ns < kShortWaitNs ? prefill_attn_kernel<D, true> : prefill_attn_kernel<D, false>;
  if (!opt_in_smem(reinterpret_cast<const void*>(kfn), Layout<D>::ALLOC)) return ORTHRUS_ECUDA;
  return launch_kernel(kfn, dim3(static_cast<unsigned>(units)), dim3(THREADS),
                       static_cast<size_t>(Layout<D>::ALLOC), stream, tq, tk, tv, p);
}

}  // namespace pre
}  // namespace orthrus

using namespace orthrus;

extern "C" int orthrus_prefill_attn(const void* q, const orthrus_kv_cache* cache, int Hq, int P,
                                    void* out, int32_t* dev_status, void* stream) {
  if (q == nullptr || cache == nullptr || out == nullptr) return ORTHRUS_EINVAL;
  if (P < 1 || Hq < 1 || cache->B < 0 || cache->Hkv < 1) return ORTHRUS_EINVAL;
  if (Hq % cache->Hkv != 0) return ORTHRUS_ESHAPE;
  if (cache->d != 64 && cache->d != 128) return ORTHRUS_EUNSUPPORTED;
  if (cache->k == nullptr || cache->v == nullptr || cache->ctx_lens == nullptr)
    return ORTHRUS_EINVAL;
  if (cache->cap < P) return ORTHRUS_ESHAPE;
  if (static_cast<long long>(cache->B) * cache->Hkv * cache->cap >= (1ll << 31) ||
      static_cast<long long>(cache->B) * P * Hq >= (1ll << 31))
    return ORTHRUS_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(cache->k) || !aligned16(cache->v) || !aligned16(out))
    return ORTHRUS_EALIGN;
  if (cache->B == 0) return ORTHRUS_OK;
  const cudaStream_t s = as_stream(stream);
  if (cache->d == 128) return pre::launch<128>(q, cache, Hq, P, out, dev_status, s);
  return pre::launch<64>(q, cache, Hq, P, out, dev_status, s);
}
