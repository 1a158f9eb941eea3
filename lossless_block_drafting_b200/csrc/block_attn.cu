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
// G*K queries of a (sequence b, KV head g, head chunk hc) segment are packed
// into one 128-row tcgen05 M tile (row r = i*Gc + hh) and every K/V byte is
// read from HBM once.  One persistent launch of one CTA per SM (cooperative,
// or plain under programmatic dependent launch, which keeps every CTA
// resident too: see the launch);
// the keys of each segment are cut into 64-key tiles, loaded in groups of two
// (one 128-row TMA box per 128-byte column chunk).
//
// Partition.  When the segments fit the grid (S <= SMs) every CTA works
// inside one segment: segment s gets CTAs in proportion to its tiles.  By
// default a CTA streams a static run of about 3/4 of its fair share of the
// segment's groups and then claims the rest one group at a time from the
// segment's claim counter (dynamic balance: siblings finish within about one
// group of each other); ORTHRUS_ATTN_DETERMINISTIC gives every CTA a fixed
// range instead.  With more segments than CTAs the flat tile range is split
// evenly (stream-K) and a CTA may cross segments, emitting one partial result
// per segment piece.
//
// Roles (12 warps), each single-thread role on its own mbarrier ring:
//   warp 0      computes the CTA's schedule from ctx_lens (lane-parallel
//               scans), publishes the CTA's load groups as items of a ring
//               in shared memory (every other role replays the same list),
//               TMA-loads the Q tile of each piece and K into 3 stages.
//   warp 2      TMA-loads V into 3 stages; the whole warp allocates and frees
//               TMEM (all 512 columns).
//   warp 1      tcgen05 issuer of S = Q K^T, one N = 128 sequence per group
//               into one of two 128-column TMEM S buffers.
//   warp 3      tcgen05 issuer of O_w += P V, P read from TMEM (the bf16 P of
//               a tile overwrites its S columns), V an MN-major smem operand.
//   warps 4-11  two softmax warpgroups on alternate tiles, one thread per
//               row: S from TMEM, tail masking only on tail tiles, exp2
//               against a running reference max (O is rescaled only when the
//               max grows by more than 2^8, exact because the final
//               normaliser uses the same reference), P back into TMEM.  At a
//               piece end the two groups merge their (m, l, O) and write the
//               piece's fp32 partial result.
// Merge.  Per-segment partition: each CTA adds to its segment's completion
// counter once its partial is written; the segment's own CTAs then fold an
// equal share of its rows by log-sum-exp (bulk copies of the pieces' rows
// into the idle K/V ring) and write bf16.  Stream-K: a bounded grid barrier,
// then every CTA merges an equal share of all output rows.  The whole
// operation is one launch.
#include <cuda_bf16.h>

#include <atomic>
#include <cmath>

#include "common.cuh"
#include "host.h"

namespace orthrus {
namespace attn {

constexpr int TN = 64;        // keys per compute tile
// K and V are loaded in groups of two consecutive tiles of a segment (one
// 128-row TMA box per 128-byte column chunk); a tile without a partner (at a
// segment or CTA-range edge) comes alone in a 64-row box.  Larger boxes keep
// the TMA engines near HBM bandwidth (measured: 64-row boxes top out at about
// 80% of it, 128-row boxes near 97%).
constexpr int ROWS = 128;     // query rows per tile (tcgen05 M)
// Load groups of its static run a CTA asks L2 to prefetch while it still waits
// for the previous kernel in the stream (2 groups = 128 KB of K and V at D = 128;
// measured in the decode step: 2 beat 0 and 4).
constexpr int PREFETCH_GROUPS = 2;
// Balanced mode: the claim pool's last TAIL_HALF_GROUPS * cn / 2 groups (cn =
// the segment's CTAs) are handed out as single 64-key tiles.  Measured in the
// decode step (40960 x K 32): 0, i.e. whole groups to the end, is fastest; a
// lone tile costs a ring item, an S sequence and a softmax pass for half the
// keys, more than the tighter finish it buys (1 cost 0.4 us, 2 cost 0.9 us).
constexpr int TAIL_HALF_GROUPS = 0;
// Balanced mode: each CTA first streams a static run of STATIC_NUM / STATIC_DEN
// of its fair share of the segment's groups, then claims.
constexpr int STATIC_NUM = 3, STATIC_DEN = 4;
// Partial O layout: [ROWS / BR row blocks][slot][D / 4 column quads][BR rows][4]
// floats.  A warp's store of one column quad for its 32 rows covers four whole
// 128-byte lines, and since the pieces of a segment occupy consecutive slots,
// one row block of all of them is one contiguous range: the merge fetches it
// with a single bulk copy.
constexpr int BR = 8;
constexpr int THREADS = 384;  // 12 warps: TMA, MMA, TMEM alloc, spare, 2 softmax groups
constexpr int TMEM_COLS = 512;
// TMEM columns: two S buffers of 2 * TN fp32 columns, one per load group in
// flight (S of a group is one N = 128 MMA sequence; tile h of the group owns
// columns [h * TN, (h + 1) * TN) and its bf16 P overwrites the first TN / 2 of
// them), then the two softmax groups' O accumulators.
constexpr int NSB = 2;
constexpr int SBUF_COLS = 2 * TN;
constexpr int TMEM_O = NSB * SBUF_COLS;  // O_0 at 256, O_1 at 384

// The producer warp publishes the CTA's load groups, in order, as items of a
// ring in shared memory: int4 {first tile | flags << 25, L of the sequence,
// flat segment index, first cache row of the (sequence, KV head)}.
constexpr int RING = 16;
constexpr int kItemFlagShift = 25;
constexpr int kItemTileMask = (1 << kItemFlagShift) - 1;
constexpr int kItemPair = 1;        // two tiles (else one)
constexpr int kItemPieceFirst = 2;  // first group of a piece (load its Q)
constexpr int kItemPieceLast = 4;   // last group of a piece (publish its partial)
constexpr int kItemEnd = 8;         // last group of the CTA
constexpr int kItemNone = 16;       // the CTA has no group at all

template <int D>
struct Layout {
  static constexpr int CHUNKS = D / 64;            // 128-byte column chunks of a row
  static constexpr int NK = D == 128 ? 3 : 6;      // K ring stages (released after S = Q K^T)
  static constexpr int NV = NK;                    // V ring stages (released after O += P V)
  static constexpr int Q_CHUNK = ROWS * 128;
  static constexpr int KV_CHUNK = 2 * TN * 128;    // one chunk of a two-tile group
  static constexpr int HALF = TN * 128;            // offset of the group's second tile
  static constexpr int Q_BYTES = CHUNKS * Q_CHUNK;
  static constexpr int KV_BYTES = CHUNKS * KV_CHUNK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr int OFF_ML = OFF_V + NV * KV_BYTES;  // [ROWS] float2 handed WG1 -> WG0
  static constexpr int OFF_SCHED = OFF_ML + ROWS * 8;  // 9 x int64 CTA schedule
  static constexpr int OFF_ITEMS = OFF_SCHED + 128;  // RING x int4 work items
  static constexpr int OFF_BAR = OFF_ITEMS + RING * 16;
  static constexpr int NBAR = 2 * NK + 2 * NV + 15 + RING;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;        // room to align the base to 1024
};

static_assert(RING > Layout<64>::NK + NSB + 1 && RING > Layout<128>::NK + NSB + 1,
              "work-item ring must outlast the pipeline depth");

struct Params {
  const int32_t* ctx_lens;
  float* part_o;      // [ROWS / 8][slots][D / 4][8][4] unnormalised O of each piece
  float2* part_ml;    // [slots][ROWS] (m in log2 units, l)
  unsigned long long* gbar;  // grid-barrier arrival ticket counter (starts at 0)
  unsigned long long* seg_cnt;  // [SMs] per-segment completion counters (start at 0)
  unsigned long long* seg_next; // [SMs] per-segment group claim counters (0 between calls)
  __nv_bfloat16* out; // [B, K, Hq, D]
  int32_t* dev_status;
  unsigned long long wait_ns;  // bounded-wait limit
  int B, K, Hq, Hkv, G, Gc, nhc, cap, mask_mode;
  int slots;          // pieces the workspace holds (segments + grid size)
  int balance;        // per-segment partition: claim the tail groups dynamically
  float sl2;          // softmax scale * log2(e)
};

// a * b / c for non-negative operands, with 32-bit division whenever the
// product and divisor fit (64-bit division is emulated and costly).
__device__ __forceinline__ long long mul_div(long long a, long long b, long long c) {
  const unsigned long long prod = static_cast<unsigned long long>(a) * static_cast<unsigned long long>(b);
  if ((prod >> 32) == 0 && (static_cast<unsigned long long>(c) >> 32) == 0)
    return static_cast<unsigned int>(prod) / static_cast<unsigned int>(c);
  return static_cast<long long>(prod / static_cast<unsigned long long>(c));
}

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

__device__ __forceinline__ void cursor_next(Cursor& c, const Params& p) {
  if (++c.t < c.nt) return;
  c.t = 0;
  const int nseg = p.Hkv * p.nhc;
  if (++c.seg < nseg) return;
  c.seg = 0;
  c.base += static_cast<long long>(nseg) * c.nt;
  if (++c.b < p.B) cursor_load(c, p);
}

// Load groups: a group starts at an even tile of a segment (or at the CTA's
// first tile) and ends at an odd tile, the segment's last tile or the CTA's
// last tile.  Every role derives the same groups from the same cursor.
__device__ __forceinline__ bool group_first(const Cursor& c, int j) {
  return j == 0 || (c.t & 1) == 0;
}
__device__ __forceinline__ bool group_last(const Cursor& c, int j, int n) {
  return j == n - 1 || (c.t & 1) == 1 || c.t + 1 == c.nt;
}

// Work partition over P CTAs.  When the segments fit (S <= P), every CTA
// works inside a single segment: segment s gets 1 + floor((P - S) * n_s / T)
// CTAs (the first P - sum of those segments get one more) and splits its n_s
// tiles evenly among them, so no CTA pays for a mid-range piece boundary
// (pipeline drain, partial write, Q reload).  With more segments than CTAs
// the flat tile range is split evenly (stream-K style) and a CTA may cross
// segments.  Both kernels derive the same partition from ctx_lens.
__device__ __forceinline__ bool segment_partition(const Params& p, int P) {
  return static_cast<long long>(p.B) * p.Hkv * p.nhc <= P;
}

// First tile of CTA c when T tiles are split over P CTAs.
__device__ __forceinline__ long long cta_start(long long c, long long T, long long P) {
  return mul_div(c, T, P);
}
// The CTA whose range contains tile x (the last c with cta_start(c) <= x).
__device__ __forceinline__ long long cta_of(long long x, long long T, long long P) {
  return mul_div((x + 1) * P - 1, 1, T);
}

// Under the per-segment partition: the CTA's segment (flat index), its CTAs
// [c0, c0 + cn), its tiles ns and the sequence's clamped context length L.
struct OwnSeg {
  long long s;
  int c0, cn, ns, L;
};

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}
// Exclusive prefix sum over the lanes of a warp.
__device__ __forceinline__ int warp_excl_scan(int v, int lane) {
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, o);
    if (lane >= o) x += y;
  }
  return x - v;
}

// CTA c's work record, computed by the 32 lanes of one warp (sequences spread
// over the lanes, running prefix sums by warp scans); the lane that owns CTA
// c's sequence writes sched[0..8]:
//   [0], [1]  flat tile range [x0, x1)
//   [2]..[5]  the cursor at x0 (base, b | seg, t | L, nt)
//   [6]..[8]  the CTA's segment under the per-segment partition (s, or -1;
//             c0 | cn; L | ns)
// Per-segment partition (S <= P): sequence b's segments get e_b = 1 +
// floor((P - S) * n_b / T) CTAs each, the first P - sum of those segments one
// more, and a CTA splits its segment's tiles evenly with its siblings.
// Stream-K (S > P): the flat range of T tiles is split evenly.  All counts
// fit in 32 bits (B * Hkv * cap < 2^31 is checked on the host).
__device__ void warp_schedule(const Params& p, int P, int c, int lane, bool report_errors,
                              long long* sched);

// Up to 32 sequences: one load per lane and interleaved scans, no second pass.
__device__ __forceinline__ void write_sched(long long* sched, int x0, int x1, int TTx, int b,
                                            int sg, int nb, int L, int s_own, int c0, int cn) {
  sched[0] = x0;
  sched[1] = x1;
  sched[2] = TTx;
  sched[3] = (static_cast<long long>(b) << 32) | static_cast<unsigned int>(sg);
  sched[4] = (static_cast<long long>(x0 - TTx - sg * nb) << 32) | static_cast<unsigned int>(L);
  sched[5] = nb;
  sched[6] = s_own;
  sched[7] = (static_cast<long long>(c0) << 32) | static_cast<unsigned int>(cn);
  sched[8] = (static_cast<long long>(L) << 32) | static_cast<unsigned int>(nb);
}

// `raw` is lane b's ctx_lens[b] (0 for lanes >= B).
__device__ void warp_schedule_small(const Params& p, int P, int c, int lane, bool report_errors,
                                    long long* sched, int raw) {
  const int nseg = p.Hkv * p.nhc;
  const int S = p.B * nseg;
  const bool in = lane < p.B;
  if (report_errors && in && (raw < 0 || raw > p.cap - p.K)) report(p.dev_status, ORTHRUS_ECAPACITY);
  const int L = in ? clamp_len(raw, p) : 0;
  const int nb = in ? n_tiles(L, p) : 0;
  const int u = nseg * nb;
  const int T = warp_sum(u);
  const bool segp = S <= P;
  const int e = (in && segp) ? 1 + static_cast<int>(mul_div(P - S, nb, T)) : 0;
  const int v = nseg * e;
  int iv = v, iu = u;  // inclusive scans of v (CTAs) and u (tiles), interleaved
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yv = __shfl_up_sync(0xFFFFFFFFu, iv, o);
    const int yu = __shfl_up_sync(0xFFFFFFFFu, iu, o);
    if (lane >= o) {
      iv += yv;
      iu += yu;
    }
  }
  const int rem = P - __shfl_sync(0xFFFFFFFFu, iv, 31);  // < S
  const int Cx = iv - v, TTx = iu - u;
  bool found = false;
  if (in) {
    if (segp) {
      const int bs = lane * nseg;
      const int lo = Cx + min(bs, rem);
      const int hi = Cx + v + min(bs + nseg, rem);
      if (c >= lo && c < hi) {
        found = true;
        const int rb = max(0, min(nseg, rem - bs));  // segments of b with one more CTA
        const int local = c - lo;
        int sg, k, cn;
        if (local < rb * (e + 1)) {
          sg = local / (e + 1);
          k = local - sg * (e + 1);
          cn = e + 1;
        } else {
          const int l2 = local - rb * (e + 1);
          sg = rb + l2 / e;
          k = l2 - (sg - rb) * e;
          cn = e;
        }
        const int Ts = TTx + sg * nb;
        write_sched(sched, Ts + static_cast<int>(mul_div(k, nb, cn)),
                    Ts + static_cast<int>(mul_div(k + 1, nb, cn)), TTx, lane, sg, nb, L,
                    bs + sg, c - k, cn);
      }
    } else {
      const int x0s = static_cast<int>(mul_div(c, T, P)), x1s = static_cast<int>(mul_div(c + 1, T, P));
      if (x1s > x0s && x0s >= TTx && x0s < TTx + u) {
        found = true;
        write_sched(sched, x0s, x1s, TTx, lane, (x0s - TTx) / nb, nb, L, -1, 0, 0);
      }
    }
  }
  if (!__any_sync(0xFFFFFFFFu, found) && lane == 0) {  // no tiles for this CTA
    for (int i = 0; i < 9; ++i) sched[i] = 0;
    sched[6] = -1;
  }
}

__device__ void warp_schedule(const Params& p, int P, int c, int lane, bool report_errors,
                              long long* sched) {
  if (p.B <= 32) {
    warp_schedule_small(p, P, c, lane, report_errors, sched,
                        lane < p.B ? __ldcg(p.ctx_lens + lane) : 0);
    return;
  }
  const int nseg = p.Hkv * p.nhc;
  const int S = p.B * nseg;
  int tl = 0;
  for (int b = lane; b < p.B; b += 32) {
    const int raw = __ldg(p.ctx_lens + b);
    if (report_errors && (raw < 0 || raw > p.cap - p.K)) report(p.dev_status, ORTHRUS_ECAPACITY);
    tl += nseg * n_tiles(clamp_len(raw, p), p);
  }
  const int T = warp_sum(tl);
  const bool segp = S <= P;
  int rem = 0;
  if (segp) {
    int vl = 0;
    for (int b = lane; b < p.B; b += 32)
      vl += nseg * (1 + static_cast<int>(mul_div(P - S, n_tiles(clamp_len(__ldg(p.ctx_lens + b), p), p), T)));
    rem = P - warp_sum(vl);  // < S
  }
  const int x0s = static_cast<int>(mul_div(c, T, P)), x1s = static_cast<int>(mul_div(c + 1, T, P));
  bool found = false;
  int Cb = 0, TTb = 0;  // CTAs and tiles of the sequences before this chunk
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int b = b0 + lane;
    const bool in = b < p.B;
    const int L = in ? clamp_len(__ldg(p.ctx_lens + b), p) : 0;
    const int nb = in ? n_tiles(L, p) : 0;
    const int e = in ? 1 + static_cast<int>(mul_div(P - S, nb, T)) : 0;
    const int v = segp ? nseg * e : 0;
    const int u = nseg * nb;
    const int Cx = Cb + warp_excl_scan(v, lane), TTx = TTb + warp_excl_scan(u, lane);
    if (in) {
      int x0 = -1, x1 = 0, sg = 0, s_own = -1, c0 = 0, cn = 0;
      if (segp) {
        const int bs = b * nseg;
        const int lo = Cx + min(bs, rem);
        const int hi = Cx + v + min(bs + nseg, rem);
        if (c >= lo && c < hi) {
          const int rb = max(0, min(nseg, rem - bs));  // segments of b with one more CTA
          const int local = c - lo;
          int k;
          if (local < rb * (e + 1)) {
            sg = local / (e + 1);
            k = local - sg * (e + 1);
            cn = e + 1;
          } else {
            const int l2 = local - rb * (e + 1);
            sg = rb + l2 / e;
            k = l2 - (sg - rb) * e;
            cn = e;
          }
          const int Ts = TTx + sg * nb;
          x0 = Ts + static_cast<int>(mul_div(k, nb, cn));
          x1 = Ts + static_cast<int>(mul_div(k + 1, nb, cn));
          s_own = bs + sg;
          c0 = c - k;
        }
      } else if (x1s > x0s && x0s >= TTx && x0s < TTx + u) {
        sg = (x0s - TTx) / nb;
        x0 = x0s;
        x1 = x1s;
      }
      if (x0 >= 0) {
        found = true;
        sched[0] = x0;
        sched[1] = x1;
        sched[2] = TTx;
        sched[3] = (static_cast<long long>(b) << 32) | static_cast<unsigned int>(sg);
        sched[4] = (static_cast<long long>(x0 - TTx - sg * nb) << 32) | static_cast<unsigned int>(L);
        sched[5] = nb;
        sched[6] = s_own;
        sched[7] = (static_cast<long long>(c0) << 32) | static_cast<unsigned int>(cn);
        sched[8] = (static_cast<long long>(L) << 32) | static_cast<unsigned int>(nb);
      }
    }
    Cb += warp_sum(v);
    TTb += warp_sum(u);
  }
  if (!__any_sync(0xFFFFFFFFu, found) && lane == 0) {  // no tiles for this CTA
    for (int i = 0; i < 9; ++i) sched[i] = 0;
    sched[6] = -1;
  }
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

// Grid-wide barrier of a cooperative launch (all CTAs resident), split into
// arrive and wait so a CTA can do independent work in between.  Thread 0 of
// each CTA takes a ticket from a 64-bit counter that only ever grows by
// nctas per launch (so it stays a multiple of nctas between launches and
// never needs resetting); the generation is complete once the counter reaches
// the next multiple.  Bounded: a wait that gives up reports ETIMEOUT.
// grid_wait compares by signed difference, so a counter that wraps past 2^64
// still reaches its target.  Release on arrival (the CTA barrier before it
// orders the other threads' writes), acquire by the polling load.
__device__ __forceinline__ unsigned long long grid_arrive(unsigned long long* gbar,
                                                          unsigned int nctas) {
  fence_acq_rel_gpu();
  const unsigned long long ticket = atomicAdd(gbar, 1ull);
  return (ticket / nctas + 1) * nctas;
}

__device__ bool grid_wait(unsigned long long* gbar, unsigned long long target,
                          int32_t* status, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  bool ok = true;
  for (uint32_t polls = 0; static_cast<long long>(ld_acquire_gpu(gbar) - target) < 0; ++polls) {
    if ((polls & 255u) == 255u && globaltimer_ns() - t0 > limit_ns) {
      report(status, ORTHRUS_ETIMEOUT);
      ok = false;
      break;
    }
  }
  return ok;
}

// CTAs [*c0, *c1] may hold pieces of segment s = (b, seg); *tall is the flat
// tile total in stream-K mode or -1 under the per-segment partition.
__device__ void segment_ctas(const Params& p, int P, int b, int seg, long long* c0,
                             long long* c1, long long* tall, int* ntb) {
  const int nseg = p.Hkv * p.nhc;
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
  *ntb = nt_b;
  *c0 = cta_of(Ts, T, P);
  *c1 = cta_of(Ts + nt_b - 1, T, P);
  *tall = T;
}

// Pieces of one segment, as seen by the merge: CTAs [c0, c1]; when `dense`
// every one of them wrote a piece, otherwise empty CTAs are skipped (tall is
// the flat tile total in stream-K mode or -1 under the per-segment partition).
struct SegPieces {
  long long c0, c1, tall;
  int ntb, dense;
};

__device__ SegPieces segment_pieces(const Params& p, int P, long long s) {
  const int nseg = p.Hkv * p.nhc;
  SegPieces sp;
  segment_ctas(p, P, static_cast<int>(s / nseg), static_cast<int>(s % nseg), &sp.c0, &sp.c1,
               &sp.tall, &sp.ntb);
  if (sp.tall >= 0)
    sp.dense = sp.tall >= P;                    // stream-K: no empty CTA at all
  else
    sp.dense = (sp.c1 - sp.c0 + 1) <= sp.ntb;  // no more CTAs than tiles
  return sp;
}

constexpr int MERGE_SEGS = 64;  // segment records precomputed per CTA

// Merge the pieces of output rows [r0, r1) (flat over segments x rows of a
// segment) by log-sum-exp; one warp per row, lane owns D/32 columns, up to 12
// pieces' loads in flight per round.  Segment records for the CTA's rows are
// in `segs` (first segment s_first, n_segs of them); rows beyond them fall
// back to computing the record in lane 0.
template <int D>
__device__ void merge_rows(const Params& p, int P, long long r0, long long r1, int warp,
                           int nwarps, int lane, const SegPieces* segs, long long s_first,
                           int n_segs) {
  constexpr int PER = D / 32;
  constexpr int BATCH = 12;
  const int nseg = p.Hkv * p.nhc;
  const int RV = p.Gc * p.K;
  for (long long q = r0 + warp; q < r1; q += nwarps) {
    const long long s = mul_div(q, 1, RV);
    const int r = static_cast<int>(q - s * RV);
    const int b = static_cast<int>(s / nseg), seg = static_cast<int>(s % nseg);
    const int g = seg / p.nhc, hc = seg % p.nhc;
    const int i = r / p.Gc, hh = r % p.Gc;
    if (hc * p.Gc + hh >= p.G) continue;
    SegPieces sp;
    if (s - s_first < n_segs) {
      sp = segs[s - s_first];
    } else {
      SegPieces t{};
      if (lane == 0) t = segment_pieces(p, P, s);
      sp.c0 = __shfl_sync(0xFFFFFFFFu, t.c0, 0);
      sp.c1 = __shfl_sync(0xFFFFFFFFu, t.c1, 0);
      sp.tall = __shfl_sync(0xFFFFFFFFu, t.tall, 0);
      sp.ntb = __shfl_sync(0xFFFFFFFFu, t.ntb, 0);
      sp.dense = __shfl_sync(0xFFFFFFFFu, t.dense, 0);
    }
    auto has_piece = [&](long long c) {
      if (sp.dense) return true;
      if (sp.tall >= 0) return cta_start(c, sp.tall, P) != cta_start(c + 1, sp.tall, P);
      const long long k = c - sp.c0, cn = sp.c1 - sp.c0 + 1;
      return mul_div(k, sp.ntb, cn) != mul_div(k + 1, sp.ntb, cn);
    };
    float m = -INFINITY, l = 0.f;
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
    for (long long base = sp.c0; base <= sp.c1; base += BATCH) {
      float2 ml[BATCH];
      float v[BATCH][PER];
#pragma unroll
      for (int k = 0; k < BATCH; ++k) {
        const long long c = base + k;
        const bool live = c <= sp.c1 && has_piece(c);
        ml[k] = live ? __ldcg(&p.part_ml[(s + c) * ROWS + r]) : make_float2(-INFINITY, 0.f);
        // partial O layout: [ROWS / BR][slot][D / 4 column quads][BR][4]
        const float* src =
            p.part_o + ((((r / BR) * static_cast<long long>(p.slots) + s + c) * (D / 4) +
                         lane * PER / 4) * BR + r % BR) * 4 + (lane * PER) % 4;
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
      }
      float mr = m;
#pragma unroll
      for (int k = 0; k < BATCH; ++k) mr = fmaxf(mr, ml[k].x);
      if (mr != -INFINITY) {
        const float a = (m == -INFINITY) ? 0.f : fast_exp2(m - mr);
        l *= a;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] *= a;
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
          const float wk = (ml[k].x == -INFINITY) ? 0.f : fast_exp2(ml[k].x - mr);
          l += wk * ml[k].y;
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[e] += wk * v[k][e];
        }
        m = mr;
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int h = g * p.G + hc * p.Gc + hh;
    __nv_bfloat16* dst =
        p.out + ((static_cast<long long>(b) * p.K + i) * p.Hq + h) * D + lane * PER;
#pragma unroll
    for (int e = 0; e < PER; e += 2)
      *reinterpret_cast<__nv_bfloat162*>(dst + e) =
          __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
  }
}

// Per-segment partition: CTA k of the cn CTAs of segment s merges the row
// blocks of [row0, row1) of that segment (row0 is a multiple of BR), one block
// per round, the pieces in batches of up to NPB.  Lane 0 of warp 0 fetches the
// block of every piece of the batch with ONE bulk copy (no multicast); at the
// same time warp 1 + rr takes row rr: its lanes load the pieces' (m, l),
// reduce the row's running maximum and normaliser with shuffles and store each
// piece's weight.  Then thread (row, column quad) adds up its pieces' weighted
// partials and writes its four output columns as bf16.  `buf` is the idle
// K/V ring.
template <int D, bool kShortWait>
__device__ void merge_segment(const Params& p, const OwnSeg own, int row0, int row1,
                              uint8_t* buf, volatile int* abort_flag) {
  constexpr int Q4 = D / 4;                 // float4 column quads of a row
  constexpr int BLK = BR * D * 4;           // bytes of one row block of one piece
  constexpr int HEAD = 4096;                // mbarrier, weights, scales
  constexpr int AVAIL = (Layout<D>::NK + Layout<D>::NV) * Layout<D>::KV_BYTES - HEAD;
  constexpr int NPB = AVAIL / BLK < 96 ? AVAIL / BLK : 96;  // pieces per batch
  static_assert(NPB >= 32 && 64 + BR * NPB * 4 + 2 * BR * 4 <= HEAD && BR * Q4 <= THREADS &&
                    (1 + BR) * 32 <= THREADS,
                "merge staging");
  const uint32_t bar = smem_u32(buf);
  float* wt = reinterpret_cast<float*>(buf + 64);             // [BR][NPB] piece weights
  float* rs = wt + BR * NPB;                                  // [BR] rescale of the running sum
  float* rinv = rs + BR;                                      // [BR] 1 / normaliser
  const float4* o_s = reinterpret_cast<const float4*>(buf + HEAD);  // [NPB][Q4][BR]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // A wait of this CTA gave up: the status is set and nothing is merged.  The
  // second barrier keeps a later wait from raising the flag before every
  // thread has read it.
  const bool skip = *abort_flag != 0;
  __syncthreads();
  if (skip) return;
  const bool dense = p.balance || own.cn <= own.ns;  // every CTA wrote a (maybe empty) piece
  auto live = [&](int j) {
    return dense || mul_div(j, own.ns, own.cn) != mul_div(j + 1, own.ns, own.cn);
  };
  const int nseg = p.Hkv * p.nhc;
  const int s_own = static_cast<int>(own.s);  // < grid size
  const int b = s_own / nseg, seg = s_own - b * nseg;
  const int g = seg / p.nhc, hc = seg - g * p.nhc;
  const int tr = threadIdx.x % BR, tq = threadIdx.x / BR;  // this thread's (row, quad)
  const int rr = warp - 1;                                  // the row of warps 1..BR
  const long long slot0 = own.s + own.c0;
  uint32_t phase = 0;
  for (int rb = row0; rb < row1; rb += BR) {
    const int row = rb + tr;
    const bool on = tq < Q4 && row < row1;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float M = -INFINITY, L = 0.f;  // running (max, normaliser) of row rb + rr (warps 1..BR)
    for (int j0 = 0; j0 < own.cn; j0 += NPB) {
      const int nb = own.cn - j0 < NPB ? own.cn - j0 : NPB;
      if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, nb * BLK);
        fence_proxy_async_global();  // the partials were written by generic stores
        bulk_load(bar + HEAD,
                  p.part_o + (static_cast<long long>(rb / BR) * p.slots + slot0 + j0) * (BLK / 4),
                  nb * BLK, bar);
      } else if (rr >= 0 && rr < BR) {
        // lane l holds pieces l, l + 32, ... of the batch (all loads in flight)
        constexpr int PL = (NPB + 31) / 32;
        const bool row_on = rb + rr < row1;
        float2 mlr[PL];
        float mb = M;
#pragma unroll
        for (int u = 0; u < PL; ++u) {
          const int j = lane + 32 * u;
          mlr[u] = (j < nb && row_on && live(j0 + j))
                       ? __ldcg(p.part_ml + (slot0 + j0 + j) * ROWS + rb + rr)
                       : make_float2(-INFINITY, 0.f);
          mb = fmaxf(mb, mlr[u].x);
        }
        for (int o = 16; o > 0; o >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xFFFFFFFFu, mb, o));
        float lsum = 0.f;
#pragma unroll
        for (int u = 0; u < PL; ++u) {
          const int j = lane + 32 * u;
          // empty or dead pieces weigh 0 (their partial O is never read)
          const float w = mlr[u].x == -INFINITY ? 0.f : fast_exp2(mlr[u].x - mb);
          if (j < nb) wt[rr * NPB + j] = w;
          lsum += w * mlr[u].y;
        }
        for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xFFFFFFFFu, lsum, o);
        const float sc = (M == -INFINITY || mb == -INFINITY) ? 0.f : fast_exp2(M - mb);
        L = L * sc + lsum;
        M = mb;
        if (lane == 0) {
          rs[rr] = sc;
          rinv[rr] = L > 0.f ? 1.f / L : 0.f;
        }
      }
      // A wait that gives up still lets the copy land before the CTA leaves
      // (it targets this CTA's shared memory); then every thread returns.
      if (!mbar_wait_bounded<kShortWait>(bar, phase, abort_flag, p.dev_status, p.wait_ns))
        mbar_wait_drain(bar, phase, p.dev_status);
      phase ^= 1u;
      __syncthreads();
      if (*abort_flag) return;  // read by all threads between the same two barriers
      if (on) {
        const float sc = rs[tr];
        acc.x *= sc;
        acc.y *= sc;
        acc.z *= sc;
        acc.w *= sc;
        for (int jj = 0; jj < nb; ++jj) {
          const float w = wt[tr * NPB + jj];
          if (w == 0.f) continue;  // empty or dead piece: its partial may be stale
          const float4 x = o_s[(jj * Q4 + tq) * BR + tr];
          acc.x += w * x.x;
          acc.y += w * x.y;
          acc.z += w * x.z;
          acc.w += w * x.w;
        }
      }
      __syncthreads();
    }
    if (on) {
      const int i = row / p.Gc, hh = row % p.Gc;
      if (hc * p.Gc + hh < p.G) {
        const float inv = rinv[tr];
        const int h = g * p.G + hc * p.Gc + hh;
        __nv_bfloat16* dst =
            p.out + ((static_cast<long long>(b) * p.K + i) * p.Hq + h) * D + tq * 4;
        uint2 pk;
        pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2*>(dst) = pk;
      }
    }
  }
}

template <int D, bool kShortWait>
__global__ void __launch_bounds__(THREADS, 1)
    attn_splitkv_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK2,
                        const __grid_constant__ CUtensorMap tmK1,
                        const __grid_constant__ CUtensorMap tmV2,
                        const __grid_constant__ CUtensorMap tmV1, const Params p) {
  using Ly = Layout<D>;
  constexpr int NK = Ly::NK;
  constexpr int NV = Ly::NV;
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
  auto s_full = [&](int i) { return bar2 + 8u * (2 + i); };   // S of buffer i ready
  auto sb_free = [&](int i) { return bar2 + 8u * (4 + i); };  // P*V done with buffer i
  auto p_full = [&](int i) { return bar2 + 8u * (6 + i); };   // P of buffer i / 2, half i & 1
  const uint32_t o_full = bar2 + 8u * 10;
  const uint32_t o_free = bar2 + 8u * 11;
  const uint32_t mma_done = bar2 + 8u * 12;  // both MMA issuers commit once at exit
  // piece epilogue hand-offs between the softmax groups (bounded waits, so a
  // group that gave up never leaves the other one stuck at a barrier)
  const uint32_t xchg_ml = bar2 + 8u * 13;      // WG1's (m, l) are in ml_xchg
  const uint32_t xchg_scale = bar2 + 8u * 14;   // WG0's two scales are in ml_xchg
  auto item_full = [&](int i) { return bar2 + 8u * (15 + i); };  // work item i published
  int4* items = reinterpret_cast<int4*>(smem + Ly::OFF_ITEMS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Ly::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Ly::OFF_MISC + 4);
  float2* ml_xchg = reinterpret_cast<float2*>(smem + Ly::OFF_ML);

  // Programmatic dependent launch: the next kernel in the stream may be
  // scheduled now; its CTAs land on SMs as this grid's CTAs exit (one CTA
  // fills an SM's shared memory).  Everything a preceding kernel may write
  // (ctx_lens, q, the cache, the workspace, dev_status) is touched only after
  // grid_dep_wait.
  grid_dep_launch();
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK2);
    prefetch_tmap(&tmK1);
  } else if (threadIdx.x == 64) {
    prefetch_tmap(&tmV2);
    prefetch_tmap(&tmV1);
  }

  // The CTA's tile range and its starting cursor are computed by warp 0 and
  // shared, while warp 1 initialises the barriers.
  long long* sched = reinterpret_cast<long long*>(smem + Ly::OFF_SCHED);

  const int nseg = p.Hkv * p.nhc;
  // Per-segment partition: this CTA's segment (s = -1 in stream-K mode),
  // read where it is needed rather than kept live through the tile loops.
  auto read_own = [&]() {
    const volatile long long* sv = sched;
    return OwnSeg{sv[6], static_cast<int>(sv[7] >> 32), static_cast<int>(sv[7] & 0xffffffff),
                  static_cast<int>(sv[8] & 0xffffffff), static_cast<int>(sv[8] >> 32)};
  };
  auto read_start = [&]() {
    Cursor c;
    c.base = sched[2];
    c.b = static_cast<int>(sched[3] >> 32);
    c.seg = static_cast<int>(sched[3] & 0xffffffff);
    c.t = static_cast<int>(sched[4] >> 32);
    c.L = static_cast<int>(sched[4] & 0xffffffff);
    c.nt = static_cast<int>(sched[5]);
    return c;
  };

  // ---------------------------------------- work list, Q and K producer
  // Thread 0 decides the CTA's load groups (up to two 64-key tiles of one
  // segment), publishes each as an item of the shared ring (every other role
  // replays the same list) and issues the Q tile of each piece and the
  // group's K.  produce(limit) emits groups until `limit` have been emitted
  // or the list ends; it runs once before the prologue barrier (the first NK
  // groups need no free stage, so HBM traffic starts right after the
  // schedule) and resumes in the producer role.
  int pr_gi = 0, pr_pieces = 0;
  OwnSeg pr_own{-1, 0, 0, 0, 0};
  Cursor pr_c{};
  int pr_n = 0, pr_j = 0, pr_cur = -2;
  int pr_sg = 0, pr_sg_end = 0, pr_pool0 = 0, pr_ngr = 0, pr_gclaims = 0, pr_tile0 = 0;
  bool pr_grabbing = false, pr_dry = true;
  unsigned long long pr_pend = 0;
  const uint64_t pr_policy = policy_evict_first();
  int pr_s = -1, pr_kvbase = 0, pr_qh = 0, pr_qb = 0;  // cached for the current segment
  auto emit = [&](int t, int L, int s, int flags) -> bool {
    const int slot = pr_gi % RING;
    if (s != pr_s && s >= 0) {
      pr_s = s;
      const int b = s / nseg, seg = s - b * nseg;
      const int g = seg / p.nhc, hc = seg - g * p.nhc;
      pr_kvbase = (b * p.Hkv + g) * p.cap;
      pr_qh = g * p.G + hc * p.Gc;
      pr_qb = b * p.K;
    }
    const int kvbase = pr_kvbase;
    // Ring slots are never overwritten early: the producer is at most NK
    // groups ahead of S = Q K^T, which is at most NSB groups ahead of P V,
    // which trails every other reader of an item (RING > NK + NSB + 1).
    items[slot] = make_int4(t | (flags << kItemFlagShift), L, s, kvbase);
    mbar_arrive(item_full(slot));
    if (flags & kItemNone) return true;
    if (flags & kItemPieceFirst) {
      if (!mbar_try_wait(q_empty, (pr_pieces & 1) ^ 1) &&
          !mbar_wait_bounded<kShortWait>(q_empty, (pr_pieces & 1) ^ 1, abort_flag, p.dev_status,
                                         p.wait_ns))
        return false;
      mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(p.Gc * p.K * D * 2));
      for (int c = 0; c < Ly::CHUNKS; ++c)
        tma_load_3d(sb0 + Ly::OFF_Q + c * Ly::Q_CHUNK, &tmQ, q_full, c * 64, pr_qh, pr_qb);
      ++pr_pieces;
    }
    const bool pair = flags & kItemPair;
    const int stage = pr_gi % NK;
    if (!mbar_try_wait(empty_k(stage), ((pr_gi / NK) & 1) ^ 1) &&
        !mbar_wait_bounded<kShortWait>(empty_k(stage), ((pr_gi / NK) & 1) ^ 1, abort_flag,
                                       p.dev_status, p.wait_ns))
      return false;
    mbar_arrive_expect_tx(full_k(stage), (pair ? 2 : 1) * Ly::HALF * Ly::CHUNKS);
    for (int c = 0; c < Ly::CHUNKS; ++c)
      tma_load_2d_hint(sb0 + Ly::OFF_K + stage * Ly::KV_BYTES + c * Ly::KV_CHUNK,
                       pair ? &tmK2 : &tmK1, full_k(stage), c * 64, kvbase + t * TN, pr_policy);
    ++pr_gi;
    return true;
  };
  // Balanced per-segment partition: the CTA first streams a static run of
  // about 3/4 of its fair share of the segment's 128-key groups, then claims
  // groups of the remaining pool one at a time from the segment's claim
  // counter (the next claim is always in flight, so its latency is hidden,
  // and siblings finish within about one group of each other).  The counter
  // is 0 when a call starts: the segment's last CTA puts it back to 0 once
  // every sibling has finished claiming (see the merge below).
  auto start_claims = [&]() {
    pr_pend = atomicAdd(p.seg_next + pr_own.s, 1ull);
    pr_grabbing = true;
  };
  // Work units are (first tile << 1) | pair.  The static run and the claims
  // are 128-key groups (the pool's last TAIL_HALF_GROUPS * cn / 2 groups, if
  // any, as single 64-key tiles).
  auto group_unit = [&](int g) { return (4 * g) | (2 * g + 1 < pr_own.ns ? 1 : 0); };
  auto next_unit = [&]() -> int {
    if (pr_sg < pr_sg_end) {
      const int g = pr_sg++;
      if (!pr_grabbing && !pr_dry && pr_sg_end - pr_sg <= 1) start_claims();
      return group_unit(g);
    }
    if (pr_dry) return -1;
    if (!pr_grabbing) start_claims();
    const long long c = static_cast<long long>(pr_pend);
    int u;
    if (c < pr_gclaims) {
      u = group_unit(pr_pool0 + static_cast<int>(c));
    } else {
      const long long t = pr_tile0 + (c - pr_gclaims);
      if (t >= pr_own.ns) {
        pr_dry = true;
        return -1;
      }
      u = static_cast<int>(t) << 1;
    }
    pr_pend = atomicAdd(p.seg_next + pr_own.s, 1ull);  // next claim, in flight
    return u;
  };
  // Before the barrier (pre) no other role runs yet, so only groups that need
  // no wait are emitted: the first NK (fresh K stages) of the first piece.
  auto produce = [&](int limit, bool pre) {
    if (pr_own.s >= 0 && p.balance) {
      if (pr_cur == -2) {
        pr_cur = next_unit();
        if (pr_cur < 0) emit(0, pr_own.L, static_cast<int>(pr_own.s), kItemNone);
      }
      while (pr_cur >= 0 && pr_gi < limit) {
        const int nxt = next_unit();
        const bool pair = pr_cur & 1;
        const int flags = (pair ? kItemPair : 0) | (pr_gi == 0 ? kItemPieceFirst : 0) |
                          (nxt < 0 ? (kItemPieceLast | kItemEnd) : 0);
        if (!emit(pr_cur >> 1, pr_own.L, static_cast<int>(pr_own.s), flags)) {
          pr_cur = -1;
          break;
        }
        pr_cur = nxt;
      }
    } else {
      // Static range [x0, x0 + n) of the flat tile space (deterministic).
      if (pr_cur == -2) {
        pr_cur = 0;
        if (pr_n == 0) emit(0, 0, static_cast<int>(pr_own.s), kItemNone);
      }
      while (pr_j < pr_n && pr_gi < limit) {
        const bool pair = !group_last(pr_c, pr_j, pr_n);
        const int jl = pr_j + (pair ? 1 : 0);
        const bool pfirst = (pr_j == 0) || pr_c.t == 0;
        const bool plast = (jl == pr_n - 1) || pr_c.t + (pair ? 1 : 0) == pr_c.nt - 1;
        const int flags = (pair ? kItemPair : 0) | (pfirst ? kItemPieceFirst : 0) |
                          (plast ? kItemPieceLast : 0) | (jl == pr_n - 1 ? kItemEnd : 0);
        if (pre && pfirst && pr_pieces > 0) break;  // its Q waits for the previous piece's
        if (!emit(pr_c.t, pr_c.L, pr_c.b * nseg + pr_c.seg, flags)) {
          pr_j = pr_n;
          break;
        }
        cursor_next(pr_c, p);
        if (pair) cursor_next(pr_c, p);
        pr_j = jl + 1;
      }
    }
  };

  if (threadIdx.x == 32) {
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
    for (int i = 0; i < NSB; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(sb_free(i), 1);
      mbar_init(p_full(2 * i), 4);
      mbar_init(p_full(2 * i + 1), 4);
    }
    mbar_init(o_full, 1);
    mbar_init(o_free, 8);
    mbar_init(mma_done, 2);
    mbar_init(xchg_ml, 4);
    mbar_init(xchg_scale, 4);
    for (int i = 0; i < RING; ++i) mbar_init(item_full(i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  {
    // Query rows past the Gc*K real ones are never loaded: zero them once so
    // their scores are plain zeros (whole 128-byte rows, swizzle-invariant).
    const int first_pad = p.Gc * p.K;
    const int pieces16 = (ROWS - first_pad) * 8 * Ly::CHUNKS;
    for (int q = threadIdx.x; q < pieces16; q += THREADS) {
      const int ch = q / ((ROWS - first_pad) * 8), rem = q % ((ROWS - first_pad) * 8);
      *reinterpret_cast<uint4*>(smem + Ly::OFF_Q + ch * Ly::Q_CHUNK +
                                (first_pad + rem / 8) * 128 + (rem % 8) * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }

  // L2 warm-up while the previous kernel drains.  Warp 0 guesses the CTA's
  // first static load groups from the lengths as they read now (through L2
  // only, so no line of them stays in L1 past the wait) and prefetches their
  // K and V into L2.  A prefetch moves nothing into shared memory and writes
  // nothing, so a stale length (one that kernel is still changing) or a wrong
  // guess costs bandwidth, never a result; the schedule itself is computed
  // again after the wait.  Rows past the cache view are dropped by the tensor
  // map's bounds.
  int raw_pre = 0;        // lane b: ctx_lens[b] as read before the wait
  bool have_pre = false;  // the schedule in shared memory was computed from raw_pre
  if (warp == 0 && p.B <= 32 && p.balance) {
    raw_pre = lane < p.B ? __ldcg(p.ctx_lens + lane) : 0;
    warp_schedule_small(p, gridDim.x, blockIdx.x, lane, false, sched, raw_pre);
    have_pre = true;
    __syncwarp();
    if (lane == 0) {
      const OwnSeg g0 = read_own();
      if (g0.s >= 0 && g0.cn > 0) {
        const int k = static_cast<int>(blockIdx.x) - g0.c0;
        const int fs = static_cast<int>(
            mul_div(STATIC_NUM * ((g0.ns + 1) / 2), 1, STATIC_DEN * g0.cn));
        const int b = static_cast<int>(g0.s) / nseg, seg = static_cast<int>(g0.s) - b * nseg;
        const int kvbase = (b * p.Hkv + seg / p.nhc) * p.cap;
        const int n = fs < PREFETCH_GROUPS ? fs : PREFETCH_GROUPS;
        for (int i = 0; i < n; ++i) {
          const int row = kvbase + 2 * (k * fs + i) * TN;
          for (int c = 0; c < Ly::CHUNKS; ++c) {
            tma_prefetch_2d(&tmK2, c * 64, row);
            tma_prefetch_2d(&tmV2, c * 64, row);
          }
        }
      }
    }
    __syncwarp();
  }

  grid_dep_wait();
  if (warp == 0) {
    if (have_pre) {
      // The schedule is a function of the lengths alone: if every length reads
      // as it did before the wait, the one already in shared memory stands.
      const int raw = lane < p.B ? __ldcg(p.ctx_lens + lane) : 0;
      if (__all_sync(0xFFFFFFFFu, raw == raw_pre)) {
        if (blockIdx.x == 0 && lane < p.B && (raw < 0 || raw > p.cap - p.K))
          report(p.dev_status, ORTHRUS_ECAPACITY);
      } else {
        warp_schedule_small(p, gridDim.x, blockIdx.x, lane, blockIdx.x == 0, sched, raw);
      }
    } else {
      warp_schedule(p, gridDim.x, blockIdx.x, lane, blockIdx.x == 0, sched);
    }
    __syncwarp();
  }
  // warps 0 and 1 meet: the barriers are initialised and the schedule written
  if (warp < 2) asm volatile("bar.sync 2, 64;" ::: "memory");
  if (threadIdx.x == 0) {
    pr_own = read_own();
    pr_c = read_start();
    pr_n = static_cast<int>(sched[1] - sched[0]);
    if (pr_own.s >= 0 && p.balance) {
      const int k = static_cast<int>(blockIdx.x) - pr_own.c0;
      pr_ngr = (pr_own.ns + 1) / 2;
      const int fs = static_cast<int>(mul_div(STATIC_NUM * pr_ngr, 1, STATIC_DEN * pr_own.cn));
      pr_pool0 = pr_own.cn * fs;
      pr_sg = k * fs;
      pr_sg_end = pr_sg + fs;
      pr_dry = pr_pool0 >= pr_ngr;
      const int pool = pr_ngr - pr_pool0;             // groups left to claim
      const int tail = (TAIL_HALF_GROUPS * pr_own.cn + 1) / 2;  // groups cut into tiles
      pr_gclaims = pool > tail ? pool - tail : 0;
      pr_tile0 = 2 * (pr_pool0 + pr_gclaims);         // then tiles from here
    }
    produce(NK, true);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

#define WAIT_OR(barrier, parity, on_fail) \
  if (!mbar_wait_bounded<kShortWait>((barrier), (parity), abort_flag, p.dev_status, p.wait_ns)) on_fail
#define WARP_WAIT_OR(barrier, parity, on_fail) \
  if (!mbar_wait_warp<kShortWait>((barrier), (parity), abort_flag, p.dev_status, p.wait_ns)) on_fail

  if (warp == 0 && lane == 0) {
    // ------------------------------------ work list, Q and K producer
    // (its first NK groups were issued before the prologue barrier)
    produce(1 << 30, false);
    // Drain: every issued copy must have landed before the CTA may exit.
    for (int q = (pr_gi > NK ? pr_gi - NK : 0); q < pr_gi; ++q)
      mbar_wait_drain(full_k(q % NK), (q / NK) & 1, p.dev_status);
    if (pr_pieces > 0) mbar_wait_drain(q_full, (pr_pieces - 1) & 1, p.dev_status);
  } else if (warp == 2 && lane == 0) {
    // ------------------------------------------------------- V producer
    const uint64_t policy = policy_evict_first();
    int gi = 0;
    for (;;) {
      const int slot = gi % RING;
      WAIT_OR(item_full(slot), (gi / RING) & 1, break);
      const int4 it = items[slot];
      const int flags = it.x >> kItemFlagShift;
      if (flags & kItemNone) break;
      const int t = it.x & kItemTileMask;
      const bool pair = flags & kItemPair;
      const int stage = gi % NV;
      WAIT_OR(empty_v(stage), ((gi / NV) & 1) ^ 1, break);
      mbar_arrive_expect_tx(full_v(stage), (pair ? 2 : 1) * Ly::HALF * Ly::CHUNKS);
      for (int c = 0; c < Ly::CHUNKS; ++c)
        tma_load_2d_hint(sb0 + Ly::OFF_V + stage * Ly::KV_BYTES + c * Ly::KV_CHUNK,
                         pair ? &tmV2 : &tmV1, full_v(stage), c * 64, it.w + t * TN, policy);
      ++gi;
      if (flags & kItemEnd) break;
    }
    for (int q = (gi > NV ? gi - NV : 0); q < gi; ++q)
      mbar_wait_drain(full_v(q % NV), (q / NV) & 1, p.dev_status);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------ S = Q K^T issuer
    // One N = 128 (or 64 for a lone tile) MMA sequence per load group into
    // TMEM buffer g % 2; the buffer is reused once P*V of group g - 2 is done.
    // Descriptors are built once; per group only the stage offset is added.
    const uint32_t id_s2 = make_idesc_bf16_f32(ROWS, 2 * TN, false, false);
    const uint32_t id_s1 = make_idesc_bf16_f32(ROWS, TN, false, false);
    uint64_t qd[D / 16], kd[D / 16];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      qd[kk] = make_sdesc(sb0 + Ly::OFF_Q + (kk >> 2) * Ly::Q_CHUNK + (kk & 3) * 32, 16, 1024,
                          kSwizzle128B);
      kd[kk] = make_sdesc(sb0 + Ly::OFF_K + (kk >> 2) * Ly::KV_CHUNK + (kk & 3) * 32, 16, 1024,
                          kSwizzle128B);
    }
    int q_seen = 0, gi = 0;
    for (;;) {
      const int slot = gi % RING;
      WAIT_OR(item_full(slot), (gi / RING) & 1, break);
      const int flags = items[slot].x >> kItemFlagShift;
      if (flags & kItemNone) break;
      if (flags & kItemPieceFirst) {
        WAIT_OR(q_full, q_seen & 1, break);
        ++q_seen;
      }
      const int stage = gi % NK;
      const int gb = gi & 1;
      WAIT_OR(full_k(stage), (gi / NK) & 1, break);
      if (gi >= NSB) {
        WAIT_OR(sb_free(gb), ((gi >> 1) - 1) & 1, break);
      }
      tc_fence_after();
      const uint64_t koff = static_cast<uint64_t>((stage * Ly::KV_BYTES) >> 4);
      const uint32_t id = (flags & kItemPair) ? id_s2 : id_s1;
      const uint32_t dst = tmem + gb * SBUF_COLS;
      mma_bf16_ss(dst, qd[0], kd[0] + koff, id, 0u);
#pragma unroll
      for (int kk = 1; kk < D / 16; ++kk) mma_bf16_ss(dst, qd[kk], kd[kk] + koff, id, 1u);
      mma_commit(empty_k(stage));
      mma_commit(s_full(gb));
      if (flags & kItemPieceLast) mma_commit(q_empty);
      ++gi;
      if (flags & kItemEnd) break;
    }
    // every MMA of both issuers must be complete before TMEM is released
    mma_commit(mma_done);
    mbar_wait_drain(mma_done, 0, p.dev_status);
  } else if (warp == 3 && lane == 0) {
    // ------------------------------------------------ O_w += P V issuer
    const uint32_t id_pv = make_idesc_bf16_f32(ROWS, D, false, true);
    uint64_t vd[TN / 16];
#pragma unroll
    for (int kk = 0; kk < TN / 16; ++kk)
      // V is [keys x d] with d contiguous: MN-major B operand; 16 keys per step
      // = two 8-row swizzle atoms (2048 B); d chunks Ly::KV_CHUNK apart.
      vd[kk] = make_sdesc(sb0 + Ly::OFF_V + kk * 2048, Ly::KV_CHUNK, 1024, kSwizzle128B);
    int pieces_done = 0, jp = 0, gi = 0, j = 0;
    uint32_t pf_par = 0;  // bit pb: parity of P barrier pb's next phase (kept in a register)
    bool fail = false;
    for (;;) {
      const int slot = gi % RING;
      WAIT_OR(item_full(slot), (gi / RING) & 1, break);
      const int flags = items[slot].x >> kItemFlagShift;
      if (flags & kItemNone) break;
      if (flags & kItemPieceFirst) {
        jp = j;
        if (pieces_done > 0) {
          WAIT_OR(o_free, (pieces_done - 1) & 1, break);
        }
      }
      const int gb = gi & 1, stage = gi % NV;
      const int ntl = (flags & kItemPair) ? 2 : 1;
      for (int h = 0; h < ntl; ++h, ++j) {
        const int w = j & 1;
        const int pb = 2 * gb + h;
        WAIT_OR(p_full(pb), (pf_par >> pb) & 1u, { fail = true; break; });
        pf_par ^= 1u << pb;
        if (h == 0) {
          WAIT_OR(full_v(stage), (gi / NV) & 1, { fail = true; break; });
        }
        tc_fence_after();
        const uint64_t voff = static_cast<uint64_t>((stage * Ly::KV_BYTES + h * Ly::HALF) >> 4);
        const uint32_t a_p = tmem + gb * SBUF_COLS + h * TN;  // P: 16 keys = 8 columns
        const uint32_t dst = tmem + TMEM_O + w * 128;
        const bool fresh = (j - jp) < 2;  // first tile of group w in this piece
        mma_bf16_ts(dst, a_p, vd[0] + voff, id_pv, fresh ? 0u : 1u);
#pragma unroll
        for (int kk = 1; kk < TN / 16; ++kk)
          mma_bf16_ts(dst, a_p + kk * 8, vd[kk] + voff, id_pv, 1u);
      }
      if (fail) break;
      mma_commit(empty_v(stage));
      mma_commit(sb_free(gb));
      if (flags & kItemPieceLast) {
        mma_commit(o_full);
        ++pieces_done;
      }
      ++gi;
      if (flags & kItemEnd) break;
    }
    mma_commit(mma_done);
    mbar_wait_drain(mma_done, 0, p.dev_status);
  } else if (warp >= 4) {
    // ------------------------------------------------ softmax + epilogue
    const int w = (warp - 4) >> 2;            // softmax warpgroup: even / odd tiles
    const int r = (warp & 3) * 32 + lane;     // query row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t t_o = lane_base + TMEM_O + w * 128;
    const int rows_valid = p.Gc * p.K;
    const int i_row = r / p.Gc;
    const bool idle_warp = (warp & 3) * 32 >= rows_valid;
    const float sl2 = p.sl2;
    int pieces = 0, jp = 0, gi = 0, j = 0, prev_gi = 0;
    float m_used = -INFINITY, l_sum = 0.f;
    bool fail = false;
#define FAIL          \
  {                   \
    fail = true;      \
    break;            \
  }
    // A tile that runs past the valid keys: the warpgroup's 128 threads zero
    // those V rows together, so that stale or NaN cache contents cannot reach
    // O through 0 * NaN.  Returns false if the V stage never arrived.
    auto zero_v_tail = [&](int tile0, int kv_end, bool first_half) -> bool {
      const int stage = gi % NV;
      if (!mbar_wait_warp<kShortWait>(full_v(stage), (gi / NV) & 1, abort_flag, p.dev_status, p.wait_ns))
        return false;
      const int nv = kv_end - tile0 > 0 ? kv_end - tile0 : 0;
      const int per_chunk = (TN - nv) * 8;
      uint8_t* vt = smem + Ly::OFF_V + stage * Ly::KV_BYTES + (first_half ? 0 : Ly::HALF);
      for (int q = r; q < per_chunk * Ly::CHUNKS; q += ROWS) {
        const int ch = q / per_chunk, rem = q % per_chunk;
        *reinterpret_cast<uint4*>(vt + ch * Ly::KV_CHUNK + (nv + rem / 8) * 128 +
                                  (rem % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      return true;
    };
    for (;;) {
      const int slot = gi % RING;
      WARP_WAIT_OR(item_full(slot), (gi / RING) & 1, break);
      const int2 itxy = *reinterpret_cast<const int2*>(&items[slot]);
      const int flags = itxy.x >> kItemFlagShift;
      if (flags & kItemNone) {
        // No group at all: publish an empty piece (its m = -inf) for the merge.
        const int s_it = items[slot].z;
        if (w == 0 && s_it >= 0 && r < rows_valid)
          p.part_ml[(static_cast<long long>(s_it) + blockIdx.x) * ROWS + r] =
              make_float2(-INFINITY, 0.f);
        break;
      }
      const int t0 = itxy.x & kItemTileMask;
      const int Lc = itxy.y;
      const int ntl = (flags & kItemPair) ? 2 : 1;
      if (flags & kItemPieceFirst) {
        jp = j;
        m_used = -INFINITY;
        l_sum = 0.f;
      }
      // Tile h of the group is tile j + h of the CTA; warpgroup w takes the
      // tiles with (j + h) & 1 == w: at most one per group.
      const int h = (w - j) & 1;
      const int jt = j + h;
      j += ntl;
      if (h < ntl) do {
        if (idle_warp) {
          // All 32 rows of this warp are padding: no softmax, but it still
          // waits for S (which keeps it within one phase of the P barriers),
          // takes its share of a tail tile's V zeroing, and arrives so the P*V
          // issuer's count is complete.  The P rows it leaves unwritten feed
          // only padding rows of O, which are never read.
          WARP_WAIT_OR(s_full(gi & 1), (gi >> 1) & 1, FAIL);
          const int tile0 = (t0 + h) * TN;
          const int kv_end = Lc + p.K;
          if (tile0 + TN > kv_end && !zero_v_tail(tile0, kv_end, h == 0)) FAIL;
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full(2 * (gi & 1) + h));
          prev_gi = gi;
          break;
        }
        const bool fresh = (jt - jp) < 2;
        const int gb = gi & 1;
        const int half = h;
        const uint32_t t_s = lane_base + gb * SBUF_COLS + half * TN;
        const int kv_end = Lc + p.K;
        const int tile0 = (t0 + h) * TN;
        WARP_WAIT_OR(s_full(gb), (gi >> 1) & 1, FAIL);
        tc_fence_after();
        // p = 2^(s*sl2 - m) against the running reference m (scale and shift as
        // packed f32x2 FMAs, exp2 on the SFU, row sum as packed adds).  Pass 0
        // is the common case; the first tile of a piece takes its own max
        // first.  Every p is positive, so a tile row sum of at most 2^8 proves
        // no element exceeded the reference by more than 2^8: only otherwise
        // (rare) does pass 1 reload S, take the tile max, rescale O_w and l
        // and redo the tile.  One copy of the tile code keeps the hot loop
        // small in the instruction cache.
        const float2 sc2 = make_float2(sl2, sl2);
        float x[TN];
        float2 acc2[4];
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
          uint32_t sr[TN];
          tmem_ld64(t_s, sr);
          tmem_wait_ld();
          if (tile0 + TN > Lc + 1) {
            // Tail tile: some keys lie past some row's limit.  Interior tiles
            // (every key < L + 1) skip this entirely.
            const int lim = (r >= rows_valid) ? 0
                            : (p.mask_mode == ORTHRUS_MASK_DIFF ? kv_end : Lc + i_row + 1);
#pragma unroll
            for (int c = 0; c < TN; ++c)
              if (tile0 + c >= lim) sr[c] = __float_as_uint(-INFINITY);
          }
          const bool take_max = fresh || pass == 1;
          if (take_max) {
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < TN; c += 8) {
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
              // O_w may only be touched once this group's previous P*V (tile
              // j - 2, in load group prev_gi) has completed.
              WARP_WAIT_OR(sb_free(prev_gi & 1), (prev_gi >> 1) & 1, FAIL);
              tc_fence_after();
#pragma unroll
              for (int c0 = 0; c0 < D; c0 += 16) {
                uint32_t o[16];
                tmem_ld16(t_o + c0, o);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
                tmem_st16(t_o + c0, o);
              }
              tmem_wait_st();
              l_sum *= f;
              m_used = m_new;
            }
          }
          // each S value is read once, so S and P are never both live in registers
          const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
          const float2 nm2 = make_float2(-m_eff, -m_eff);
#pragma unroll
          for (int q = 0; q < 4; ++q) acc2[q] = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < TN; c += 2) {
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

        if (tile0 + TN > kv_end && !zero_v_tail(tile0, kv_end, h == 0)) FAIL;
        uint32_t pk[TN / 2];
#pragma unroll
        for (int c = 0; c < TN / 2; ++c) pk[c] = pack_bf16x2(x[2 * c], x[2 * c + 1]);
        tmem_st32(t_s, pk);  // P over the first TN / 2 columns of its S buffer
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(2 * gb + half));
        prev_gi = gi;
      } while (0);
      if (fail) break;

      if (flags & kItemPieceLast) {
        // Piece epilogue: merge the two groups' (m, l, O) and publish it.  WG1
        // hands its (m, l) to WG0 (xchg_ml), which writes the row's (M, l) and
        // hands back the two scales in the same slot (xchg_scale); then each
        // group writes half of the columns.  Thread r of each group is the
        // only reader and writer of ml_xchg[r] on its side, and each side
        // writes only after the other side's hand-off, so one slot suffices.
        WARP_WAIT_OR(o_full, pieces & 1, break);
        tc_fence_after();
        const long long pslot = static_cast<long long>(items[slot].z) + blockIdx.x;
        float a0, a1;
        if (w == 1) {
          ml_xchg[r] = make_float2(m_used, l_sum);
          __syncwarp();
          if (lane == 0) mbar_arrive(xchg_ml);
          WARP_WAIT_OR(xchg_scale, pieces & 1, break);
          const float2 sc = ml_xchg[r];
          a0 = sc.x;
          a1 = sc.y;
        } else {
          WARP_WAIT_OR(xchg_ml, pieces & 1, break);
          const float2 o1 = ml_xchg[r];
          const float M = fmaxf(m_used, o1.x);
          a0 = (m_used == -INFINITY) ? 0.f : fast_exp2(m_used - M);
          a1 = (o1.x == -INFINITY) ? 0.f : fast_exp2(o1.x - M);
          if (!idle_warp) p.part_ml[pslot * ROWS + r] = make_float2(M, a0 * l_sum + a1 * o1.y);
          ml_xchg[r] = make_float2(a0, a1);
          __syncwarp();
          if (lane == 0) mbar_arrive(xchg_scale);
        }
        if (!idle_warp) {  // rows of all-padding warps are never merged
          // partial O in row blocks (BR rows x D / 4 quads x 4 floats): the
          // warp's 32 rows of one column quad fill four whole lines
          float4* dst = reinterpret_cast<float4*>(p.part_o) +
                        ((r / BR) * static_cast<long long>(p.slots) + pslot) * (D / 4) * BR +
                        r % BR;
#pragma unroll
          for (int c0 = w * (D / 2); c0 < (w + 1) * (D / 2); c0 += 32) {
            uint32_t o0[32], o1r[32];
            tmem_ld32(lane_base + TMEM_O + c0, o0);
            tmem_ld32(lane_base + TMEM_O + 128 + c0, o1r);
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
              dst[((c0 + k) / 4) * BR] = v;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);  // all 8 softmax warps are done with O
        ++pieces;
      }
      ++gi;
      if (flags & kItemEnd) break;
    }
#undef FAIL
  }
#undef WAIT_OR
#undef WARP_WAIT_OR

  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }

  const int RV = p.Gc * p.K;
  const OwnSeg own = read_own();
  if (own.s >= 0) {
    // Per-segment partition: the cn CTAs of this CTA's segment each add to the
    // segment's counter once their piece is written (the first adds 2^20 -
    // (cn - 1), the rest 1, so every call adds exactly 2^20 and the counter
    // never needs a reset); a CTA's own add pins the call's target.  Then the
    // segment's rows are merged by its own CTAs, an equal share each.  All
    // siblings have added only after their last claim, so once the target is
    // reached the last CTA of the segment (which always has rows to merge)
    // puts the claim counter back to 0 for the next call.
    // shares of whole BR-row blocks (the last CTA's share is never empty)
    const int k = static_cast<int>(blockIdx.x) - own.c0;
    const int nblk = (RV + BR - 1) / BR;
    const int row0 = BR * static_cast<int>(mul_div(k, nblk, own.cn));
    const int row1e = BR * static_cast<int>(mul_div(k + 1, nblk, own.cn));
    const int row1 = row1e < RV ? row1e : RV;
    if (threadIdx.x == 0) {
      // the release covers this CTA's partial (written before the CTA barrier)
      const unsigned long long add = k == 0 ? (1ull << 20) - (own.cn - 1) : 1ull;
      const unsigned long long old = atom_add_release_gpu(p.seg_cnt + own.s, add);
      if (row1 > row0 &&
          grid_wait(p.seg_cnt + own.s, ((old >> 20) + 1) << 20, p.dev_status, p.wait_ns) &&
          k == own.cn - 1 && p.balance)
        *reinterpret_cast<volatile unsigned long long*>(p.seg_next + own.s) = 0ull;
    }
    __syncthreads();
    merge_segment<D, kShortWait>(p, own, row0, row1, smem + Ly::OFF_K, abort_flag);
    return;
  }

  // Every CTA's partials are written: meet at the grid barrier, then merge an
  // equal share of the output rows.  Thread 0 first records which CTAs hold
  // pieces of the segments of this CTA's rows (into the now idle K ring).
  const long long R = static_cast<long long>(p.B) * nseg * RV;
  const long long r0 = mul_div(blockIdx.x, R, gridDim.x);
  const long long r1 = mul_div(blockIdx.x + 1, R, gridDim.x);
  SegPieces* segs = reinterpret_cast<SegPieces*>(smem + Ly::OFF_K);
  const long long s_first = mul_div(r0, 1, RV);
  const long long s_last = r1 > r0 ? mul_div(r1 - 1, 1, RV) : s_first - 1;
  const int n_segs = static_cast<int>(s_last - s_first + 1 < MERGE_SEGS ? s_last - s_first + 1
                                                                        : MERGE_SEGS);
  if (threadIdx.x == 0) {
    const unsigned long long target = grid_arrive(p.gbar, gridDim.x);
    for (int k = 0; k < n_segs; ++k) segs[k] = segment_pieces(p, gridDim.x, s_first + k);
    grid_wait(p.gbar, target, p.dev_status, p.wait_ns);
  }
  __syncthreads();
  merge_rows<D>(p, gridDim.x, r0, r1, warp, THREADS / 32, lane, segs, s_first, n_segs);
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

// Workspace: [0, 256) the grid-barrier ticket, then `sms` 64-bit completion
// counters and `sms` 64-bit claim counters (per-segment counters exist only
// when the segments fit the grid, S <= sms, so this region has the same size
// and place for every shape), padded to 256 bytes, then the partial O and
// (m, l) of every piece.  The counters must be zero before the first use;
// after every completed call the ticket is a multiple of the grid size, each
// completion counter a multiple of 2^20 and each claim counter 0, whatever
// the shape, so one zeroed workspace serves any sequence of shapes it is large
// enough for.
constexpr size_t WS_TICKET = 256;

size_t counter_bytes(int sms) {  // completion + claim counters
  return (2 * static_cast<size_t>(sms) * sizeof(unsigned long long) + 255) / 256 * 256;
}

size_t workspace_bytes(const Shape& sh, int sms) {
  const size_t slots = static_cast<size_t>(sh.S) + static_cast<size_t>(sms);
  const size_t o_bytes = slots * ROWS * sh.d * sizeof(float);
  const size_t ml_bytes = slots * ROWS * sizeof(float2);
  return WS_TICKET + counter_bytes(sms) + o_bytes + ml_bytes;
}

template <int D>
int launch(const Shape& sh, const void* q, const orthrus_kv_cache* cache, int mask_mode,
           void* out, void* ws, int sms, int32_t* dev_status, cudaStream_t stream) {
  CUtensorMap tq;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(sh.Hq),
                              static_cast<uint64_t>(sh.B) * sh.K};
    const uint64_t strides[2] = {static_cast<uint64_t>(D) * 2,
                                 static_cast<uint64_t>(sh.Hq) * D * 2};
    const uint32_t box[3] = {64u, static_cast<uint32_t>(sh.Gc), static_cast<uint32_t>(sh.K)};
    const int rc = encode_tmap_bf16(&tq, q, 3, dims, strides, box);
    if (rc != ORTHRUS_OK) return rc;
  }
  CUtensorMap tk2, tk1, tv2, tv1;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(D),
                              static_cast<uint64_t>(sh.B) * sh.Hkv * cache->cap};
    const uint64_t strides[1] = {static_cast<uint64_t>(D) * 2};
    const uint32_t box2[2] = {64u, static_cast<uint32_t>(2 * TN)};
    const uint32_t box1[2] = {64u, static_cast<uint32_t>(TN)};
    int rc = encode_tmap_bf16(&tk2, cache->k, 2, dims, strides, box2);
    if (rc == ORTHRUS_OK) rc = encode_tmap_bf16(&tk1, cache->k, 2, dims, strides, box1);
    if (rc == ORTHRUS_OK) rc = encode_tmap_bf16(&tv2, cache->v, 2, dims, strides, box2);
    if (rc == ORTHRUS_OK) rc = encode_tmap_bf16(&tv1, cache->v, 2, dims, strides, box1);
    if (rc != ORTHRUS_OK) return rc;
  }
  Params p;
  p.ctx_lens = cache->ctx_lens;
  const size_t slots = static_cast<size_t>(sh.S) + static_cast<size_t>(sms);
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.gbar = reinterpret_cast<unsigned long long*>(w);
  p.seg_cnt = reinterpret_cast<unsigned long long*>(w + WS_TICKET);
  p.seg_next = p.seg_cnt + sms;
  const size_t head = WS_TICKET + counter_bytes(sms);
  p.part_o = reinterpret_cast<float*>(w + head);
  p.part_ml = reinterpret_cast<float2*>(w + head + slots * ROWS * D * sizeof(float));
  p.out = static_cast<__nv_bfloat16*>(out);
  p.dev_status = dev_status;
  p.wait_ns = wait_limit_ns();
  p.B = sh.B;
  p.K = sh.K;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.G = sh.G;
  p.Gc = sh.Gc;
  p.nhc = sh.nhc;
  p.slots = static_cast<int>(slots);
  p.cap = cache->cap;
  p.mask_mode = mask_mode & 1;
  p.balance = (mask_mode & ORTHRUS_ATTN_DETERMINISTIC) ? 0 : 1;
  p.sl2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));

  auto* kfn = p.wait_ns < kShortWaitNs ? attn_splitkv_kernel<D, true>
                                       : attn_splitkv_kernel<D, false>;
  if (!opt_in_smem(reinterpret_cast<const void*>(kfn), Layout<D>::ALLOC)) return ORTHRUS_ECUDA;
  // The sibling wait and the grid barrier before the merge need every CTA of
  // the grid resident at once (one CTA per SM; the shared memory allows no
  // second).  Under programmatic dependent launch the launch is plain: this
  // grid's CTAs then take SMs as the previous grid's CTAs exit, run their
  // prologue (and the L2 warm-up) there and wait (griddepcontrol.wait) before
  // they read anything that kernel may have written; a cooperative grid could
  // only start once the previous grid had left every SM.  Residency still
  // holds: every CTA triggers its dependents (griddepcontrol.launch_dependents)
  // on entry, so a later grid of the stream is scheduled only once all of this
  // grid's CTAs hold an SM, an earlier grid never waits on this one, and one
  // CTA per SM fits (checked once below).  Kernels of other streams can still
  // hold SMs while some CTAs wait for theirs; past the wait limit that ends the
  // call with ETIMEOUT.  Callers that overlap other streams' kernels with
  // attention set ORTHRUS_ATTN_COOPERATIVE (or ORTHRUS_NO_PDL): the launch is
  // then cooperative, which the runtime starts only when the whole grid fits.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sms);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = Layout<D>::ALLOC;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cudaError_t e = cudaErrorNotSupported;
  if (pdl_enabled() && !attn_cooperative()) {
    static std::atomic<int> fits{-1};  // one CTA per SM fits: checked once
    if (fits.load(std::memory_order_relaxed) < 0) {
      int per_sm = 0;
      const bool ok = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                          &per_sm, kfn, THREADS, Layout<D>::ALLOC) == cudaSuccess;
      fits.store(ok && per_sm >= 1 ? 1 : 0, std::memory_order_relaxed);
    }
    if (fits.load(std::memory_order_relaxed) == 0) return ORTHRUS_ECUDA;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kfn, tq, tk2, tk1, tv2, tv1, p);
    if (e != cudaSuccess) return ORTHRUS_ECUDA;
    return ORTHRUS_OK;
  }
  // Cooperative, with the programmatic attribute as well when it is on (the
  // prologue then overlaps only the previous kernel's final flush).  If the
  // runtime refuses the pair, the first (eager) call finds out and every later
  // call launches cooperatively only.
  static std::atomic<bool> coop_pdl_ok{true};
  const bool pair = pdl_enabled() && coop_pdl_ok.load(std::memory_order_relaxed);
  cfg.attrs = pair ? attr : attr + 1;
  cfg.numAttrs = pair ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, kfn, tq, tk2, tk1, tv2, tv1, p);
  if (e != cudaSuccess && pair) {
    (void)cudaGetLastError();
    coop_pdl_ok.store(false, std::memory_order_relaxed);
    cfg.attrs = attr + 1;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kfn, tq, tk2, tk1, tv2, tv1, p);
  }
  if (e != cudaSuccess) return ORTHRUS_ECUDA;
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
  if ((mask_mode & ~ORTHRUS_ATTN_DETERMINISTIC) != ORTHRUS_MASK_DIFF &&
      (mask_mode & ~ORTHRUS_ATTN_DETERMINISTIC) != ORTHRUS_MASK_AR)
    return ORTHRUS_EINVAL;
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
