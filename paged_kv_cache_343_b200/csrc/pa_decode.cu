// pa_decode.cu -- paged decode attention for sm_100a ("PagedAttention",
// section "How attention reads paged memory": for each query token walk the
// sequence's block table, gather each block's keys and values from the shared
// pool and run attention over them with an online softmax).
//
// Three launches per call, all on the caller's stream:
//   1. plan     (1 CTA)   the units of work ("entries": sequences, packs of
//                         sequences over a shared prompt, or chunks of a
//                         sequence's query tokens), prefix sums of their
//                         16-token tiles and the segment bookkeeping, written
//                         to the workspace;
//   2. main     (1 CTA per SM and head group, persistent)  the batch's tiles
//                         laid end to end are cut into equal shares, one per
//                         CTA; a producer warp streams each tile's K and V
//                         from the pool into shared memory with 5-D TMA loads
//                         (one block-table lookup per block), and consumer
//                         warps (one to two per KV head) compute S^T = K Q^T
//                         and O^T += V^T P^T on the tensor cores, the query
//                         heads of a KV head (and the query rows of an entry)
//                         packed into the MMA's N dimension, with an fp32
//                         online softmax;
//   3. combine            merges the (o, m, l) partials of every output row
//                         whose tiles were split across CTAs, partitions or
//                         a pack and the sequence's own tail.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cstring>
#include <mutex>
#include <vector>

#include "pa_decode_common.cuh"
#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

// ---------------------------------------------------------------------------
// plan (one CTA)
//   entries     the units of work laid end to end: first the K packs (only
//               with shared_blocks: pack j attends sequences b_j .. b_j+P-1
//               over their first pack_tiles[j] tiles, which they share), then
//               every sequence b over its remaining tiles seq_pre[b] ..
//               ceil(L_b / 16) - 1 (seq_pre[b] = 0 outside packs);
//   tiles[e]    = sum_{e' < e} (tiles of entry e')          (N = tiles[E] in all)
//   segments    an entry's tiles are cut wherever a partition starts (every
//               tiles_per_part tiles from its first tile) or a CTA's share
//               starts (lo(c) of the LineCut: floor(c N / C), or with a
//               split the packs' tiles and the sequences' tiles cut
//               separately); each piece is one segment, numbered 0, 1, ...
//               within the entry;
//   seg_base[e] = sum_{e' < e} (segments of e'), so the partials of entry e
//               occupy slots seg_base[e] .. seg_base[e + 1] - 1;
//   start_seq[c], first_k[c]: the entry holding lo(c) and the number of
//               that entry's segments that start before lo(c).
// Two ways to count, chosen by the host from the expected cut points per
// entry.  Few: each entry walks its own cut points in order.  Many (long
// sequences, partitions), with no walk over the cut points: CTA c "holds" the start lo(c)
// when its share is not empty (lo(c) < lo(c + 1)), so every distinct start
// is held once; it "coincides" when lo(c) is also a partition start of its
// entry.  With SD, SDC the prefix sums over c of held and held-and-coincident,
// and cnt(x) the number of CTAs with lo(c) < x (LineCut::count_below):
//   segments(e)  = partitions(e) + SD/SDC counts over CTAs cnt(t0) .. cnt(t1);
//   first_k[c]   = partition starts of e below lo(c) + held starts in
//                  [cnt(t0), c) - coincident ones among them.
// ---------------------------------------------------------------------------
constexpr int kPlanWarps = kPlanThreads / 32;

// Exclusive block-wide prefix sum of one value per thread; *total gets the sum.
__device__ __forceinline__ int32_t block_exclusive_scan(int32_t v, int32_t* warp_buf,
                                                        int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) warp_buf[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int32_t w = lane < kPlanWarps ? warp_buf[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += u;
    }
    if (lane < kPlanWarps) warp_buf[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int32_t before = (warp > 0 ? warp_buf[warp - 1] : 0) + inc - v;
  *total = warp_buf[kPlanWarps - 1];
  __syncthreads();  // warp_buf is reused by the next call
  return before;
}

// The same for two values per thread at once (warp_buf holds 2 kPlanWarps
// words): exclusive sums in ex[0..1], block totals in total[0..1].
__device__ __forceinline__ void block_exclusive_scan2(int32_t v0, int32_t v1, int32_t* warp_buf,
                                                      int32_t* ex, int32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t i0 = v0, i1 = v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u0 = __shfl_up_sync(0xffffffffu, i0, o);
    const int32_t u1 = __shfl_up_sync(0xffffffffu, i1, o);
    if (lane >= o) {
      i0 += u0;
      i1 += u1;
    }
  }
  if (lane == 31) {
    warp_buf[warp] = i0;
    warp_buf[kPlanWarps + warp] = i1;
  }
  __syncthreads();
  if (warp == 0) {
    int32_t w0 = lane < kPlanWarps ? warp_buf[lane] : 0;
    int32_t w1 = lane < kPlanWarps ? warp_buf[kPlanWarps + lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u0 = __shfl_up_sync(0xffffffffu, w0, o);
      const int32_t u1 = __shfl_up_sync(0xffffffffu, w1, o);
      if (lane >= o) {
        w0 += u0;
        w1 += u1;
      }
    }
    if (lane < kPlanWarps) {  // inclusive over warps
      warp_buf[lane] = w0;
      warp_buf[kPlanWarps + lane] = w1;
    }
  }
  __syncthreads();
  ex[0] = (warp > 0 ? warp_buf[warp - 1] : 0) + i0 - v0;
  ex[1] = (warp > 0 ? warp_buf[kPlanWarps + warp - 1] : 0) + i1 - v1;
  total[0] = warp_buf[kPlanWarps - 1];
  total[1] = warp_buf[2 * kPlanWarps - 1];
  __syncthreads();  // warp_buf is reused by the next call
}

// Smallest c in [0, C] with lo[c] >= x, i.e. the number of CTA shares that
// start below x (lo non-decreasing, lo[C] = N >= x).
__device__ __forceinline__ int32_t ctas_below(const int32_t* lo, int32_t C, int64_t x) {
  int32_t a = 0, z = C;  // the answer is in [a, z]
  while (a < z) {
    const int32_t mid = (a + z) >> 1;
    if (lo[mid] < x) a = mid + 1; else z = mid;
  }
  return a;
}

// Walks the segment starts of entry b (tiles [t0, t1)) in order: the
// partition starts and the CTA-share starts (lo[c]), equal points counted
// once.  Records start_seq / first_k for every CTA whose share starts inside
// b and returns the number of segments.
__device__ int32_t plan_sequence_segments(const DecodeParams& p, int32_t b, int64_t t0,
                                          int64_t t1, const int32_t* lo, int32_t C) {
  int32_t c = ctas_below(lo, C, t0);  // first CTA with lo(c) >= t0
  int64_t part = t0;                  // next partition start
  const int64_t tpp = p.tiles_per_part;
  int32_t count = 0;
  int64_t last = -1;
  while (true) {
    const int64_t cta_pt = (c < C && lo[c] < t1) ? lo[c] : INT64_MAX;
    const int64_t part_pt = part < t1 ? part : INT64_MAX;
    if (cta_pt == INT64_MAX && part_pt == INT64_MAX) break;
    if (cta_pt <= part_pt) {
      const int32_t idx = (cta_pt == last) ? count - 1 : count;
      if (cta_pt != last) { ++count; last = cta_pt; }
      p.start_seq[c] = b;
      p.first_k[c] = idx;
      ++c;
    } else {
      if (part_pt != last) { ++count; last = part_pt; }
      part = (tpp == INT_MAX) ? INT64_MAX : part + tpp;
    }
  }
  return count;
}

constexpr int kPlanSmemTiles = 4096;  // entries whose prefix sums are searched in shared memory
constexpr int kPlanMaxCtas = 2048;    // CTAs per head group the plan can describe
static_assert(kEntryWeight == PA_PLAN_ENTRY_WEIGHT && kPlanSmemTiles == PA_PLAN_WEIGHTED_MAX_ENTRIES,
              "the header states the plan's weighting");

// Largest e in [0, n) with tiles[e] <= x (tiles non-decreasing, tiles[0] = 0 <= x).
__device__ __forceinline__ int upper_entry(const int32_t* tiles, int n, int64_t x) {
  int lo = 0, hi = n;  // invariant: tiles[lo] <= x, answer in [lo, hi)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tiles[mid] <= x) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ void __launch_bounds__(kPlanThreads) pa_plan_kernel(DecodeParams p) {
  __shared__ int32_t warp_buf[2 * kPlanWarps];
  __shared__ int32_t s_tiles[kPlanSmemTiles + 1];
  // s_sd, s_sdc: the closed form's prefix sums over CTAs; before them the
  // same words hold the entries' virtual starts while the line is cut
  __shared__ int32_t s_aux[2 * (kPlanMaxCtas + 1)];
  static_assert(2 * (kPlanMaxCtas + 1) >= kPlanSmemTiles + 1, "virtual starts fit s_aux");
  int32_t* const s_sd = s_aux;
  int32_t* const s_sdc = s_aux + kPlanMaxCtas + 1;
  __shared__ int32_t s_lo[kPlanMaxCtas + 1];  // first tile of each CTA's share
  const int tid = threadIdx.x;
  const int B = p.num_seqs;
  griddep_launch_dependents();
  griddep_wait();  // seq_lens may come from the previous kernel on the stream
  int E = 0;       // entries
  const bool multi = p.q_start != nullptr;
  if (multi) {
    // ---- several query tokens per sequence: entry = a chunk of at most
    // q_per_entry consecutive query rows of one sequence; it reads the tokens
    // up to its last query's position
    const int Qc = p.q_per_entry;
    for (int r = tid; r < p.num_rows; r += kPlanThreads) p.q_entry[r] = -1;
    __syncthreads();
    int32_t ecarry = 0;
    for (int b0 = 0; b0 < B; b0 += kPlanThreads) {  // uniform trip count: the scan syncs
      const int b = b0 + tid;
      int32_t nch = 0, qlen = 0, L = 0, q0 = 0;
      if (b < B) {
        q0 = p.q_start[b];
        qlen = p.q_start[b + 1] - q0;
        const int32_t raw = p.seq_lens[b];
        if (raw < 0 || raw > p.max_seq_len || qlen < 0 || q0 < 0 ||
            static_cast<int64_t>(q0) + qlen > p.num_rows) {
          flag_error(p.err, PA_DEVERR_BAD_SEQLEN);
          qlen = (qlen < 0 || q0 < 0 || static_cast<int64_t>(q0) + qlen > p.num_rows) ? 0 : qlen;
        }
        L = clamp_len(raw, p.max_seq_len);
        nch = (qlen + Qc - 1) / Qc;
      }
      int32_t tot = 0;
      const int32_t eb = ecarry + block_exclusive_scan(nch, warp_buf, &tot);
      for (int j = 0; j < nch; ++j) {
        const int e = eb + j;
        if (e >= p.num_rows) {  // overlapping query ranges: more chunks than rows
          flag_error(p.err, PA_DEVERR_BAD_SEQLEN);
          break;
        }
        const int32_t nq = min(Qc, qlen - j * Qc);
        p.ent_b[e] = b;
        p.ent_q0[e] = q0 + j * Qc;
        p.ent_nq[e] = nq;
        p.ent_tok[e] = max(0, min(L, L - qlen + j * Qc + nq));
        for (int r = 0; r < nq; ++r) p.q_entry[q0 + j * Qc + r] = e;
      }
      ecarry += tot;
    }
    E = min(ecarry, p.num_rows);
    __syncthreads();  // the entries are read back below
  }
  // ---- packs: aligned windows b = P w .. P w + P - 1 over their shared
  // prefix; a window whose members do not all share one (or the shorter last
  // window) falls back to the aligned pairs inside it
  int K = 0;
  if (p.pack_size > 1) {
    const int PK = p.pack_size;
    const int W = (B + PK - 1) / PK;
    // prefix tiles common to sequences b0 .. b0 + n - 1 (0 if under the minimum)
    auto common_tiles = [&](int b0, int n) {
      int64_t P = INT64_MAX;  // blocks common to all members and full in each
      for (int m = 0; m < n; ++m) {
        P = min(P, static_cast<int64_t>(clamp_len(p.seq_lens[b0 + m], p.max_seq_len) /
                                        p.block_size));
        if (m + 1 < n) P = min(P, static_cast<int64_t>(max(0, p.shared_blocks[b0 + m])));
      }
      const int32_t tiles = static_cast<int32_t>(P * p.block_size / kTile);
      return tiles < kMinPackTiles ? 0 : tiles;
    };
    for (int w0 = 0; w0 < W; w0 += kPlanThreads) {  // uniform trip count: the scan syncs
      const int w = w0 + tid;
      int32_t whole = 0, npairs = 0;
      int32_t pair_tiles[kMaxPack / 2] = {0, 0, 0, 0};
      const int n = w < W ? min(PK, B - w * PK) : 0;  // sequences of this window
      if (w < W) {
        whole = n == PK ? common_tiles(w * PK, PK) : 0;
        if (whole == 0 && PK > 2) {
          for (int j = 0; j < n / 2; ++j) {
            pair_tiles[j] = common_tiles(w * PK + 2 * j, 2);
            if (pair_tiles[j] > 0) ++npairs;
          }
        }
      }
      const int32_t mine = whole > 0 ? 1 : npairs;
      int32_t count = 0;
      int32_t k = K + block_exclusive_scan(mine, warp_buf, &count);
      if (w < W) {
        const int b0 = w * PK;
        for (int m = 0; m < n; ++m) {
          p.seq_pack[b0 + m] = -1;
          p.seq_pre[b0 + m] = 0;
        }
        if (whole > 0) {
          p.pack_first[k] = b0;
          p.pack_n[k] = PK;
          p.pack_tiles[k] = whole;
          for (int m = 0; m < PK; ++m) {
            p.seq_pack[b0 + m] = k;
            p.seq_pre[b0 + m] = whole;
          }
        } else {
          for (int j = 0; j < n / 2; ++j) {
            if (pair_tiles[j] == 0) continue;
            const int bp = b0 + 2 * j;
            p.pack_first[k] = bp;
            p.pack_n[k] = 2;
            p.pack_tiles[k] = pair_tiles[j];
            p.seq_pack[bp] = p.seq_pack[bp + 1] = k;
            p.seq_pre[bp] = p.seq_pre[bp + 1] = pair_tiles[j];
            ++k;
          }
        }
      }
      K += count;
    }
    __syncthreads();  // the pack arrays are read back below
  }
  if (!multi) E = K + B;  // entries: the packs' prefixes, then the sequences
  if (tid == 0) {
    p.meta[0] = K;
    p.meta[1] = E;
  }
  const int nchunks = (E + kPlanThreads - 1) / kPlanThreads;
  // the cut weighs entry switches when the prefix sums fit in shared memory;
  // the entries' virtual starts (s_vs) are summed with their tiles
  const bool in_smem = E <= kPlanSmemTiles;
  const int64_t w = in_smem ? kEntryWeight : 0;
  int32_t* const s_vs = s_aux;
  int32_t carry = 0, total = 0, vcarry = 0;
  for (int ch = 0; ch < nchunks; ++ch) {
    const int e = ch * kPlanThreads + tid;
    int32_t nt = 0;
    if (multi) {
      if (e < E) nt = (p.ent_tok[e] + kTile - 1) / kTile;
    } else if (e < K) {
      nt = p.pack_tiles[e];
    } else if (e < E) {
      const int b = e - K;
      const int32_t raw = p.seq_lens[b];
      if (raw < 0 || raw > p.max_seq_len) flag_error(p.err, PA_DEVERR_BAD_SEQLEN);
      nt = (clamp_len(raw, p.max_seq_len) + kTile - 1) / kTile;
      if (p.pack_size > 1) nt -= p.seq_pre[b];
    }
    int32_t ex[2], tot[2];
    block_exclusive_scan2(nt, nt > 0 ? 1 : 0, warp_buf, ex, tot);
    if (e < E) p.plan_tiles[e] = carry + ex[0];
    if (e < E && in_smem) {
      s_tiles[e] = carry + ex[0];
      s_vs[e] = carry + ex[0] + static_cast<int32_t>(w) * (vcarry + ex[1]);
    }
    carry += tot[0];
    vcarry += tot[1];
  }
  if (tid == 0) {
    p.plan_tiles[E] = carry;
    if (in_smem) {
      s_tiles[E] = carry;
      s_vs[E] = static_cast<int32_t>(carry + w * vcarry);
    }
  }
  __syncthreads();  // the prefix sums are read back below
  const int64_t N = carry;
  const int C = p.ctas_per_group;
  const int32_t tpp = p.tiles_per_part;
  const int32_t* tiles = in_smem ? s_tiles : p.plan_tiles;
  // ---- the cut: CTA c's share starts at tile s_lo[c] (also cta_lo[c]).  The
  // line is cut evenly (LineCut; with a split, the packs and the sequences
  // separately) in virtual tiles, where an entry with tiles counts
  // kEntryWeight more (its switch first); each cut is then mapped back to the
  // real tile at that virtual position.  The virtual starts (s_vs, summed
  // above) take the closed form's words until that form starts; a batch whose
  // prefix sums do not fit in shared memory is cut unweighted.
  LineCut cut;
  cut.C = C;
  cut.S = p.split_ctas;
  if (w > 0) {
    cut.N = s_vs[E];
    cut.NK = p.split_ctas > 0 ? s_vs[K] : 0;
    for (int c = tid; c <= C; c += kPlanThreads) {
      const int64_t x = cut.lo(c);
      const int e = upper_entry(s_vs, E + 1, x);
      const int64_t t =
          e >= E ? N : entry_tile(x, s_vs[e], s_tiles[e], s_tiles[e + 1] - s_tiles[e], w);
      s_lo[c] = static_cast<int32_t>(t);
      p.cta_lo[c] = static_cast<int32_t>(t);
    }
  } else {
    cut.N = N;
    cut.NK = p.split_ctas > 0 ? tiles[K] : 0;
    for (int c = tid; c <= C; c += kPlanThreads) {
      s_lo[c] = static_cast<int32_t>(cut.lo(c));
      p.cta_lo[c] = s_lo[c];
    }
  }
  __syncthreads();  // s_lo is read below, and s_aux is free again
  if (!p.plan_closed) {  // few cut points per entry: walk them
    int32_t seg_carry = 0;
    for (int ch = 0; ch < nchunks; ++ch) {
      const int e = ch * kPlanThreads + tid;
      int32_t ns = 0;
      if (e < E && N > 0) {
        const int64_t t0 = tiles[e], t1 = tiles[e + 1];
        if (t1 > t0) ns = plan_sequence_segments(p, e, t0, t1, s_lo, C);
      }
      const int32_t ex = block_exclusive_scan(ns, warp_buf, &total);
      if (e < E) p.seg_base[e] = seg_carry + ex;
      seg_carry += total;
    }
    if (tid == 0) p.seg_base[E] = seg_carry;
    return;
  }
  auto lo_of = [&](int64_t c) { return static_cast<int64_t>(s_lo[c]); };
  auto cnt_below = [&](int64_t x) { return ctas_below(s_lo, C, x); };  // CTAs with lo(c) < x
  // ---- CTAs: the entry holding each share's start; held / coincident flags,
  // scanned together as held + coincident * 2^16 (C <= kPlanMaxCtas < 2^15)
  int32_t sd_carry = 0, sdc_carry = 0;
  int my_e = 0;  // the entry of CTA tid (one chunk of CTAs)
  for (int c0 = 0; c0 < C; c0 += kPlanThreads) {  // uniform trip count: the scans sync
    const int c = c0 + tid;
    int32_t flags = 0;
    if (c < C && N > 0) {
      const int64_t x = lo_of(c);
      const int e = upper_entry(tiles, E + 1, x);
      p.start_seq[c] = e;
      my_e = e;
      const bool held = x < lo_of(c + 1);
      const int64_t t0 = tiles[e];
      const bool coin = held && (tpp == INT_MAX ? x == t0 : (x - t0) % tpp == 0);
      flags = (held ? 1 : 0) + (coin ? 1 << 16 : 0);
    }
    int32_t tot = 0;
    const int32_t ex = block_exclusive_scan(flags, warp_buf, &tot);
    if (c < C) {
      s_sd[c] = sd_carry + (ex & 0xffff);
      s_sdc[c] = sdc_carry + (ex >> 16);
    }
    sd_carry += tot & 0xffff;
    sdc_carry += tot >> 16;
  }
  if (tid == 0) {
    s_sd[C] = sd_carry;
    s_sdc[C] = sdc_carry;
  }
  __syncthreads();
  // ---- entries: segment counts and their prefix sums
  int32_t seg_carry = 0;
  for (int ch = 0; ch < nchunks; ++ch) {
    const int e = ch * kPlanThreads + tid;
    int32_t ns = 0;
    if (e < E && N > 0) {
      const int64_t t0 = tiles[e], t1 = tiles[e + 1];
      if (t1 > t0) {
        const int a = cnt_below(t0), z = cnt_below(t1);
        const int64_t parts = tpp == INT_MAX ? 1 : (t1 - t0 + tpp - 1) / tpp;
        ns = static_cast<int32_t>(parts) + (s_sd[z] - s_sd[a]) - (s_sdc[z] - s_sdc[a]);
      }
    }
    const int32_t ex = block_exclusive_scan(ns, warp_buf, &total);
    if (e < E) p.seg_base[e] = seg_carry + ex;
    seg_carry += total;
  }
  // ---- CTAs: index of the segment that starts at lo(c) inside its entry
  for (int c = tid; c < C && N > 0; c += kPlanThreads) {
    const int64_t x = lo_of(c);
    if (x >= N) continue;  // no share: the main kernel returns before reading it
    const int e = C <= kPlanThreads ? my_e : upper_entry(tiles, E + 1, x);
    const int64_t t0 = tiles[e];
    const int a = cnt_below(t0);
    const int64_t pb = x == t0 ? 0 : (tpp == INT_MAX ? 1 : (x - t0 + tpp - 1) / tpp);
    p.first_k[c] = static_cast<int32_t>(pb) + (s_sd[c] - s_sd[a]) - (s_sdc[c] - s_sdc[a]);
  }
  if (tid == 0) p.seg_base[E] = seg_carry;
}

// ---------------------------------------------------------------------------
// main kernel
// ---------------------------------------------------------------------------
// kFP8: the pools hold 8-bit E4M3 codes.  Stages then carry the codes; each
// consumer lane reads exactly the code bytes of its MMA fragments from the
// swizzled stage tile with 16-byte loads and converts them in registers to
// fp16 (exact: every code is an fp16 value); the MMAs run in fp16 (kBF16 must
// be false).  To make each lane's bytes contiguous, the fp8 path permutes
//  - the k index of S^T = K Q^T: in k-step kc, lane quad q holds
//    d = 32q + 4kc + {0,1} (k = 2q, 2q+1) and d = 32q + 4kc + {2,3}
//    (k = 2q+8, 2q+9); the query fragments use the same map, so the dot
//    products are unchanged;
//  - the output rows of O^T = V^T P^T: accumulator row grp of m-tile mt is
//    d = 16 grp + 2 mt, row grp + 8 is d = 16 grp + 2 mt + 1.
//
// Query columns.  Each consumer warp owns NB blocks of 8 query columns of one
// KV head (the N of its MMAs); CG warps share a KV head, so a head has
// 8 NB CG columns.  Column c of a tile is query head c % G of sequence
// b + c / G: a sequence's own tiles use the first G columns, a pack's tiles
// one column per (member, head).
template <int D, int HG, int NB, int CG, bool kBF16, bool kFP8>
__global__ void __launch_bounds__((HG * CG + 1) * 32, 1)
    pa_decode_main_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
  static_assert(!kFP8 || (D == 128 && !kBF16), "fp8 caches: head_dim 128, fp16 MMA");
  static_assert(!kFP8 || (NB == 1 && CG == 1), "fp8 caches: one column block per head");
  static_assert(NB == 1 || NB == 2, "one or two column blocks per warp");
  constexpr int NW = HG * CG;                      // consumer warps
  constexpr int DC = D / 64;                       // 128-byte column chunks of a 16-bit row
  constexpr int DCT = kFP8 ? 1 : DC;               // 128-byte rows per (token, head) in a stage
  constexpr int KSTEPS = D / 16;                   // k16 steps of S^T = K Q^T
  constexpr int MTILES = D / 16;                   // m16 tiles of O^T = V^T P^T
  constexpr uint32_t kTileBytes = kTile * HG * D * (kFP8 ? 1 : 2);  // K (or V) bytes per stage

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int NS = p.stages;
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + static_cast<size_t>(NS) * 2 * kTileBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(info + NS);
  const uint32_t smem_base = smem_u32(smem);
  const uint32_t bar_base = smem_u32(bars);
  auto full_k = [&](int s) { return bar_base + 8u * s; };
  auto full_v = [&](int s) { return bar_base + 8u * (NS + s); };
  auto empty = [&](int s) { return bar_base + 8u * (2 * NS + s); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hg = blockIdx.y;
  const int c = p.cta_base + blockIdx.x;  // this CTA's share of the line (LineCut)
  const int B = p.num_seqs;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full_k(s), 1);
      mbar_init(full_v(s), 1);
      mbar_init(empty(s), NW);
    }
    fence_mbar_init();
  }
  if (warp == NW && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  __syncthreads();
  griddep_wait();  // the plan (and all earlier work on the stream) is complete
  // the next launch (the combine) may start now: what it reads before its
  // own wait, the plan, is complete
  griddep_launch_dependents();
  if (!host_plan_matches(p)) {  // a plan made for another shape: no work at all
    if (threadIdx.x == 0 && c == 0 && hg == 0) flag_error(p.err, PA_DEVERR_BAD_PLAN);
    return;
  }

  // entries: packs' prefixes then sequences, or query chunks (plain: the B sequences)
  const bool plain = p.pack_size == 1 && p.q_start == nullptr;
  // this CTA's share of the tile line, as the plan cut it
  const int64_t lo = p.cta_lo[c];
  const int64_t hi = p.cta_lo[c + 1];
  if (lo >= hi) return;

  if (warp == NW) {
    // ======================= producer =======================
    if (lane != 0) {
      check_pack_tables(p, lo, hi, c, lane - 1, 31);
      return;
    }
    produce_tiles<HG, DCT>(p, &tmK, &tmV, smem_base, kTileBytes, info, full_k(0), full_v(0),
                           empty(0), NS, lo, hi, c, hg, plain,
                           [](int32_t, int32_t) { return true; });
    return;
  }

  // ================ consumers: CG warps per KV head, NB column blocks each ================
  const int g = warp / CG;                    // KV head inside the group
  const int kvh = hg * HG + g;                // KV head
  const int col0 = 8 * NB * (warp - g * CG);  // first query column of this warp
  const int G = p.group;
  const int quad = lane & 3, grp = lane >> 2;
  const int TB = p.tok_box;
  const int tb_shift = TB == 16 ? 4 : (TB == 8 ? 3 : 2);

  // Per-lane row indices of the ldmatrix addresses (see the layout note in
  // the producer: rows of 128 bytes ordered [box][head][d-chunk][token]).
  auto row_of = [&](int tok, int dc) {
    return ((tok >> tb_shift) * HG * DCT + g * DCT + dc) * TB + (tok & (TB - 1));
  };
  const int mi = lane >> 3, rr = lane & 7;
  const int k_tok = rr + 8 * (mi & 1), k_chunk = mi >> 1;   // K: non-transposed
  const int v_tok = rr + 8 * (mi >> 1), v_chunk = mi & 1;   // V: transposed
  int k_row[DC], v_row[DC];
#pragma unroll
  for (int dc = 0; dc < DC; ++dc) {
    k_row[dc] = kFP8 ? 0 : row_of(k_tok, dc);
    v_row[dc] = kFP8 ? 0 : row_of(v_tok, dc);
  }
  // fp8: stage-tile rows of this lane's tokens (see kFP8 above)
  int r8_k[2] = {0, 0}, r8_v[4] = {0, 0, 0, 0};
  if constexpr (kFP8) {
    r8_k[0] = row_of(grp, 0);
    r8_k[1] = row_of(grp + 8, 0);
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) r8_v[tt] = row_of(2 * quad + (tt & 1) + 8 * (tt >> 1), 0);
  }
  // output row of accumulator element (m-tile mt, upper = rows grp + 8)
  auto d_of = [&](int mt, int upper) {
    return kFP8 ? 16 * grp + 2 * mt + upper : mt * 16 + grp + 8 * upper;
  };
  float k_scale = 1.f, v_scale = 1.f;
  if constexpr (kFP8) {
    k_scale = *p.k_scale;
    v_scale = *p.v_scale;
  }

  // query row offset (column / G) of this lane's two accumulator columns
  int cdiv[NB][2];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    cdiv[nb][0] = (col0 + 8 * nb + 2 * quad) / G;
    cdiv[nb][1] = (col0 + 8 * nb + 2 * quad + 1) / G;
  }
  uint32_t qf[NB][KSTEPS][2];
  float acc[NB][MTILES][4];
  float m_run[NB][2], l_part[NB][2];
  int stage = 0;
  uint32_t phase = 0;
  const float sl2 = p.scale_log2 * k_scale;

  for (int64_t t = lo; t < hi; ++t) {
    if (!mbar_wait(full_k(stage), phase, p.err, p.consumer_wait_ns)) break;
    const TileInfo ti = info[stage];
    const int ncol = ti.members * G;  // query columns of this tile, per KV head
    if (CG > 1 && col0 >= ncol) {
      // No column of this warp takes part (a sequence's own tiles fill only
      // the first G columns).  A warp of column group 0 always does and waits
      // for the whole stage, so the stage can be handed back at once.
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(stage));
      if (++stage == NS) { stage = 0; phase ^= 1u; }
      continue;
    }
    if (ti.flags & kNewSeq) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        // column c: query head c % G of query row qrow0 + c / G (a pack
        // member, or one of a sequence's query tokens)
        const int col = col0 + 8 * nb + grp;
        const int member = col / G;
        const uint16_t* qb =
            p.query +
            ((static_cast<int64_t>(ti.qrow0) + member) * p.num_q_heads + kvh * G +
             (col - member * G)) *
                D;
#pragma unroll
        for (int kc = 0; kc < KSTEPS; ++kc) {
          if (col < ncol) {
            // fp8: k = 2q, 2q+1 -> d = 32q + 4kc + {0,1}; k = 2q+8, 2q+9 -> + {2,3}
            const uint16_t* qp = kFP8 ? qb + 32 * quad + 4 * kc : qb + kc * 16 + quad * 2;
            qf[nb][kc][0] = *reinterpret_cast<const uint32_t*>(qp);
            qf[nb][kc][1] = *reinterpret_cast<const uint32_t*>(qp + (kFP8 ? 2 : 8));
            if (kFP8 && p.q_bf16) {  // the fp8 path multiplies in fp16
              qf[nb][kc][0] = bf16x2_to_f16x2(qf[nb][kc][0]);
              qf[nb][kc][1] = bf16x2_to_f16x2(qf[nb][kc][1]);
            }
          } else {
            qf[nb][kc][0] = 0u;
            qf[nb][kc][1] = 0u;
          }
        }
      }
    }
    if (ti.flags & kSegStart) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int mt = 0; mt < MTILES; ++mt)
          acc[nb][mt][0] = acc[nb][mt][1] = acc[nb][mt][2] = acc[nb][mt][3] = 0.f;
        m_run[nb][0] = m_run[nb][1] = -INFINITY;
        l_part[nb][0] = l_part[nb][1] = 0.f;
      }
    }
    // Both n8 blocks always run: a block whose columns are all beyond ncol
    // works on zero queries and writes nothing.  A runtime test here splits
    // the unrolled MMA loops and costs more than the work it saves.
    constexpr bool act1 = NB > 1;
    const uint32_t kbase = smem_base + static_cast<uint32_t>(stage) * 2u * kTileBytes;
    const uint32_t vbase = kbase + kTileBytes;
    // fp8: this lane's code bytes.  K: tokens grp, grp+8, d in [32q, 32q + 32)
    // (chunks 2q, 2q+1).  V: tokens 2q, 2q+1, 2q+8, 2q+9, d in [16 grp, +16).
    uint32_t kraw[2][8], vraw[4][4];
    if constexpr (kFP8) {
#pragma unroll
      for (int rr2 = 0; rr2 < 2; ++rr2) {
        const int r = r8_k[rr2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t a = kbase + static_cast<uint32_t>(r) * 128u +
                             static_cast<uint32_t>(((2 * quad + hh) ^ (r & 7)) * 16);
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(kraw[rr2][4 * hh]), "=r"(kraw[rr2][4 * hh + 1]),
                         "=r"(kraw[rr2][4 * hh + 2]), "=r"(kraw[rr2][4 * hh + 3])
                       : "r"(a));
        }
      }
      if (!mbar_wait(full_v(stage), phase, p.err, p.consumer_wait_ns)) break;
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const int r = r8_v[tt];
        const uint32_t a = vbase + static_cast<uint32_t>(r) * 128u +
                           static_cast<uint32_t>((grp ^ (r & 7)) * 16);
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(vraw[tt][0]), "=r"(vraw[tt][1]), "=r"(vraw[tt][2]), "=r"(vraw[tt][3])
                     : "r"(a));
      }
      // the codes are in registers: hand the stage back to the producer
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(stage));
    }

    // ---- S^T[16 tok x 8 columns] = K[16 x D] * Q^T[D x 8], per n8 block
    float s[NB][4];
    float s2[4] = {0.f, 0.f, 0.f, 0.f};  // one block: odd k-steps form a second chain
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) s[nb][0] = s[nb][1] = s[nb][2] = s[nb][3] = 0.f;
#pragma unroll
    for (int kc = 0; kc < KSTEPS; ++kc) {
      uint32_t a0, a1, a2, a3;
      if constexpr (kFP8) {
        a0 = e4m3x2_to_f16x2(static_cast<uint16_t>(kraw[0][kc] & 0xffffu));
        a2 = e4m3x2_to_f16x2(static_cast<uint16_t>(kraw[0][kc] >> 16));
        a1 = e4m3x2_to_f16x2(static_cast<uint16_t>(kraw[1][kc] & 0xffffu));
        a3 = e4m3x2_to_f16x2(static_cast<uint16_t>(kraw[1][kc] >> 16));
      } else {
        const int dc = kc >> 2;
        const int r = k_row[dc];
        const uint32_t chunk = static_cast<uint32_t>((2 * (kc & 3) + k_chunk) ^ (r & 7));
        ldmatrix_x4(kbase + static_cast<uint32_t>(r) * 128u + chunk * 16u, a0, a1, a2, a3);
      }
      if constexpr (NB == 1) {
        if (kc & 1) {
          mma_16816<kBF16>(s2, a0, a1, a2, a3, qf[0][kc][0], qf[0][kc][1]);
        } else {
          mma_16816<kBF16>(s[0], a0, a1, a2, a3, qf[0][kc][0], qf[0][kc][1]);
        }
      } else {
        mma_16816<kBF16>(s[0], a0, a1, a2, a3, qf[0][kc][0], qf[0][kc][1]);
        if (act1) mma_16816<kBF16>(s[1], a0, a1, a2, a3, qf[1][kc][0], qf[1][kc][1]);
      }
    }
    if constexpr (NB == 1) {
      s[0][0] += s2[0];
      s[0][1] += s2[1];
      s[0][2] += s2[2];
      s[0][3] += s2[3];
    }
    // ---- online softmax (base 2), masked by selection, per n8 block
    const uint32_t mask = static_cast<uint32_t>(ti.mask);
    const bool ok0 = (mask >> grp) & 1u, ok1 = (mask >> (grp + 8)) & 1u;
    uint32_t pb0[NB], pb1[NB], pc0[NB], pc1[NB];
    // The blocks' steps run side by side (their max reductions, exponentials
    // and transposes are independent), so their latencies overlap.
    float mx0[NB], mx1[NB];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      float* sv = s[nb];
      // columns 2q, 2q+1 see tile rows up to rel + column / G (rel = 16 when
      // every row is visible)
      const int limA = ti.rel + cdiv[nb][0], limB = ti.rel + cdiv[nb][1];
      const bool okA0 = ok0 && grp <= limA, okB0 = ok0 && grp <= limB;
      const bool okA1 = ok1 && grp + 8 <= limA, okB1 = ok1 && grp + 8 <= limB;
      sv[0] = okA0 ? sv[0] * sl2 : -INFINITY;
      sv[1] = okB0 ? sv[1] * sl2 : -INFINITY;
      sv[2] = okA1 ? sv[2] * sl2 : -INFINITY;
      sv[3] = okB1 ? sv[3] * sl2 : -INFINITY;
      mx0[nb] = fmaxf(sv[0], sv[2]);
      mx1[nb] = fmaxf(sv[1], sv[3]);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        mx0[nb] = fmaxf(mx0[nb], __shfl_xor_sync(0xffffffffu, mx0[nb], o));
        mx1[nb] = fmaxf(mx1[nb], __shfl_xor_sync(0xffffffffu, mx1[nb], o));
      }
    }
    float alpha0[NB], alpha1[NB];
    bool rescale = false;
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const float* sv = s[nb];
      const float mn0 = fmaxf(m_run[nb][0], mx0[nb]), mn1 = fmaxf(m_run[nb][1], mx1[nb]);
      alpha0[nb] = (mn0 == m_run[nb][0]) ? 1.f : ex2(m_run[nb][0] - mn0);
      alpha1[nb] = (mn1 == m_run[nb][1]) ? 1.f : ex2(m_run[nb][1] - mn1);
      rescale = rescale || alpha0[nb] != 1.f || alpha1[nb] != 1.f;
      m_run[nb][0] = mn0;
      m_run[nb][1] = mn1;
      const float p0 = (sv[0] == -INFINITY) ? 0.f : ex2(sv[0] - mn0);
      const float p1 = (sv[1] == -INFINITY) ? 0.f : ex2(sv[1] - mn1);
      const float p2 = (sv[2] == -INFINITY) ? 0.f : ex2(sv[2] - mn0);
      const float p3 = (sv[3] == -INFINITY) ? 0.f : ex2(sv[3] - mn1);
      // P in two 16-bit halves, P = hi + lo, so the P.V product keeps about
      // 16 significant bits of every weight instead of the storage type's 8 or 11.
      const uint32_t pt0 = pack2<kBF16>(p0, p1);  // P^T row grp     (columns 2q, 2q+1)
      const uint32_t pt1 = pack2<kBF16>(p2, p3);  // P^T row grp + 8
      const uint32_t pl0 =
          pack2<kBF16>(p0 - lo_to_float<kBF16>(pt0), p1 - hi_to_float<kBF16>(pt0));
      const uint32_t pl1 =
          pack2<kBF16>(p2 - lo_to_float<kBF16>(pt1), p3 - hi_to_float<kBF16>(pt1));
      l_part[nb][0] = l_part[nb][0] * alpha0[nb] + (p0 + p2);
      l_part[nb][1] = l_part[nb][1] * alpha1[nb] + (p1 + p3);
      // P^T as the B operand (k = token, n = column): transpose the 8x8 halves
      pb0[nb] = movmatrix_trans(pt0);
      pb1[nb] = movmatrix_trans(pt1);
      pc0[nb] = movmatrix_trans(pl0);
      pc1[nb] = movmatrix_trans(pl1);
    }
    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
        for (int mt = 0; mt < MTILES; ++mt) {
          acc[nb][mt][0] *= alpha0[nb];
          acc[nb][mt][1] *= alpha1[nb];
          acc[nb][mt][2] *= alpha0[nb];
          acc[nb][mt][3] *= alpha1[nb];
        }
      }
    }

    // ---- O^T[D x 8] += V^T[D x 16 tok] * P^T[16 tok x 8], per n8 block
    if (!kFP8 && !mbar_wait(full_v(stage), phase, p.err, p.consumer_wait_ns)) break;
    const bool partial = mask != 0xffffu;
    uint32_t z01 = 0xffffffffu, z23 = 0xffffffffu;
    if (partial) {
      const int tk = 2 * quad;
      z01 = (((mask >> tk) & 1u) ? 0x0000ffffu : 0u) | (((mask >> (tk + 1)) & 1u) ? 0xffff0000u : 0u);
      z23 = (((mask >> (tk + 8)) & 1u) ? 0x0000ffffu : 0u) |
            (((mask >> (tk + 9)) & 1u) ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int mt = 0; mt < MTILES; ++mt) {
      uint32_t a0, a1, a2, a3;
      if constexpr (kFP8) {
        // word mt/2 holds d = 16 grp + 2 mt + {0, 1} at bytes 2 (mt & 1) + {0, 1};
        // pair tokens (2q, 2q+1) and (2q+8, 2q+9) byte by byte
        const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
        const int w = mt >> 1;
        uint32_t lo, hi;
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(lo) : "r"(vraw[0][w]), "r"(vraw[1][w]), "r"(sel));
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(hi) : "r"(vraw[2][w]), "r"(vraw[3][w]), "r"(sel));
        a0 = e4m3x2_to_f16x2(static_cast<uint16_t>(lo & 0xffffu));
        a1 = e4m3x2_to_f16x2(static_cast<uint16_t>(lo >> 16));
        a2 = e4m3x2_to_f16x2(static_cast<uint16_t>(hi & 0xffffu));
        a3 = e4m3x2_to_f16x2(static_cast<uint16_t>(hi >> 16));
      } else {
        const int dc = mt >> 2;
        const int r = v_row[dc];
        const uint32_t chunk = static_cast<uint32_t>((2 * (mt & 3) + v_chunk) ^ (r & 7));
        ldmatrix_x4_trans(vbase + static_cast<uint32_t>(r) * 128u + chunk * 16u, a0, a1, a2, a3);
      }
      // masked tokens may hold anything (NaN included): zero them, never multiply
      a0 &= z01;
      a1 &= z01;
      a2 &= z23;
      a3 &= z23;
      mma_16816<kBF16>(acc[0][mt], a0, a1, a2, a3, pb0[0], pb1[0]);
      mma_16816<kBF16>(acc[0][mt], a0, a1, a2, a3, pc0[0], pc1[0]);
      if constexpr (NB > 1) {
        if (act1) {
          mma_16816<kBF16>(acc[1][mt], a0, a1, a2, a3, pb0[1], pb1[1]);
          mma_16816<kBF16>(acc[1][mt], a0, a1, a2, a3, pc0[1], pc1[1]);
        }
      }
    }
    if constexpr (!kFP8) {
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(stage));
    }
    if (++stage == NS) { stage = 0; phase ^= 1u; }

    if (ti.flags & kSegEnd) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        if (nb == 1 && !act1) continue;
        const int cb = col0 + 8 * nb;  // first column of the block
        float l0 = l_part[nb][0], l1 = l_part[nb][1];
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          l0 += __shfl_xor_sync(0xffffffffu, l0, o);
          l1 += __shfl_xor_sync(0xffffffffu, l1, o);
        }
        const float inv0 = l0 > 0.f ? v_scale / l0 : 0.f;
        const float inv1 = l1 > 0.f ? v_scale / l1 : 0.f;
        const int h0 = cb + 2 * quad, h1 = h0 + 1;  // this lane's two columns
        if (ti.flags & kDirect) {  // the whole attention of the entry's rows
#pragma unroll
          for (int mt = 0; mt < MTILES; ++mt) {
            const int d0 = d_of(mt, 0), d1 = d_of(mt, 1);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int h = hh ? h1 : h0;  // column: row qrow0 + h / G, head h % G
              if (h >= ncol) continue;
              const float inv = hh ? inv1 : inv0;
              const float v0 = acc[nb][mt][hh] * inv, v1 = acc[nb][mt][2 + hh] * inv;
              const int r = h / G;
              const int64_t o =
                  ((static_cast<int64_t>(ti.qrow0) + r) * p.num_q_heads + kvh * G + (h - r * G)) *
                  D;
              if (p.out_dtype == PA_F32) {
                float* op = static_cast<float*>(p.out);
                op[o + d0] = v0;
                op[o + d1] = v1;
              } else if (p.out_dtype == PA_BF16) {
                __nv_bfloat16* op = static_cast<__nv_bfloat16*>(p.out);
                op[o + d0] = __float2bfloat16_rn(v0);
                op[o + d1] = __float2bfloat16_rn(v1);
              } else {
                __half* op = static_cast<__half*>(p.out);
                op[o + d0] = __float2half_rn(v0);
                op[o + d1] = __float2half_rn(v1);
              }
            }
          }
        } else if (ti.seg < p.nseg_cap) {
          const int64_t prow = part_row(p, ti.seg, kvh, 0);
          float* po = p.part_o + prow * D;
#pragma unroll
          for (int mt = 0; mt < MTILES; ++mt) {
            const int d0 = d_of(mt, 0), d1 = d_of(mt, 1);
            if (h0 < ncol) {
              po[h0 * D + d0] = acc[nb][mt][0] * inv0;
              po[h0 * D + d1] = acc[nb][mt][2] * inv0;
            }
            if (h1 < ncol) {
              po[h1 * D + d0] = acc[nb][mt][1] * inv1;
              po[h1 * D + d1] = acc[nb][mt][3] * inv1;
            }
          }
          if (grp == 0) {
            float* pm = p.part_ml + prow * 2;
            if (h0 < ncol) {
              pm[h0 * 2] = l0 > 0.f ? m_run[nb][0] : -INFINITY;
              pm[h0 * 2 + 1] = l0;
            }
            if (h1 < ncol) {
              pm[h1 * 2] = l1 > 0.f ? m_run[nb][1] : -INFINITY;
              pm[h1 * 2 + 1] = l1;
            }
          }
        } else {
          flag_error(p.err, PA_DEVERR_BAD_SEQLEN);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// combine: out[b, h] = sum_k w_k o_k / sum_k w_k,  w_k = l_k 2^(m_k - M),
// M = max_k m_k over the partials k of sequence b: the segments of its own
// entry (slots seg_base[K + b] .., column h) and, when b belongs to pack j,
// those of the pack's entry (slots seg_base[j] .., column member * G + h).
// grid (B, ceil(Hq / kCombineWarps)), one warp per query head; the weights are
// found with the lanes spread over partials, then the lanes (spread over
// head_dim) stream the partial outputs with no dependence between partials.
// ---------------------------------------------------------------------------
// The partials of output row r, query head h (h inside its KV head's group):
// those of its own entry (slots s0 .., column col0) and, for a pack member,
// those of the pack's entry (slots s1 .., column col1).  direct: the main
// kernel wrote the row itself.  valid: the row belongs to an entry.  Read
// from L2 before the combine waits on the main kernel: the plan is complete
// once any main CTA has let the combine start.
struct RowParts {
  int32_t s0, ns, col0, s1, np, col1;
  bool direct, valid;
};

__device__ __forceinline__ RowParts row_parts(const DecodeParams& p, int r, int h) {
  RowParts q;
  q.s1 = q.np = q.col1 = 0;
  q.valid = true;
  if (p.q_start != nullptr) {  // query chunks: row r is column (r - first row) * G + h
    const int e = __ldcg(p.q_entry + r);
    q.valid = e >= 0 && e < __ldcg(p.meta + 1);
    const int ee = q.valid ? e : 0;
    q.s0 = __ldcg(p.seg_base + ee);
    q.ns = __ldcg(p.seg_base + ee + 1) - q.s0;
    q.col0 = (r - __ldcg(p.ent_q0 + ee)) * p.group + h;
    q.direct = q.ns == 1;
    return q;
  }
  const int K = p.pack_size > 1 ? __ldcg(p.meta) : 0;
  q.s0 = __ldcg(p.seg_base + K + r);
  q.ns = __ldcg(p.seg_base + K + r + 1) - q.s0;
  q.col0 = h;
  const int pk = p.pack_size > 1 ? __ldcg(p.seq_pack + r) : -1;
  q.direct = pk < 0 && q.ns == 1;
  if (pk >= 0) {
    q.s1 = __ldcg(p.seg_base + pk);
    q.np = __ldcg(p.seg_base + pk + 1) - q.s1;
    q.col1 = (r - __ldcg(p.pack_first + pk)) * p.group + h;
  }
  return q;
}

template <int D>
__global__ void __launch_bounds__(kCombineWarps * 32) pa_combine_narrow_kernel(const DecodeParams p) {
  constexpr int V = D / 32;  // floats per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int qh = blockIdx.y * kCombineWarps + warp;
  const int G = p.group;
  const int kvh = qh / G, h = qh - kvh * G;
  const bool live = qh < p.num_q_heads && host_plan_matches(p);
  RowParts rp{};
  if (live) rp = row_parts(p, b, h);  // the plan is complete: read it before the wait
  // the next launch on the stream may start its prologue now; it waits for
  // this grid before touching data
  griddep_launch_dependents();
  griddep_wait();  // the main kernel's partials are complete and visible
  if (!live || rp.direct || !rp.valid) return;  // written by the main kernel (or no entry)
  // partial k: k < ns from the row's own entry, then the pack's
  const int32_t nseq = (rp.s0 + rp.ns <= p.nseg_cap) ? rp.ns : 0;
  const int32_t npack = (rp.s1 + rp.np <= p.nseg_cap) ? rp.np : 0;
  int32_t ntot = nseq + npack;
  auto row_of = [&](int32_t k) {
    const int32_t slot = k < nseq ? rp.s0 + k : rp.s1 + (k - nseq);
    const int col = k < nseq ? rp.col0 : rp.col1;
    return part_row(p, slot, kvh, col);
  };
  const int64_t obase = (static_cast<int64_t>(b) * p.num_q_heads + qh) * D + lane * V;

  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
  float W = 0.f;
  if (ntot <= kCombineRegs) {
    // few partials: every load is issued at once, then the same arithmetic
    // in the same order as the loops below
    float mk[kCombineRegs], lk[kCombineRegs], ok[kCombineRegs][V];
#pragma unroll
    for (int k = 0; k < kCombineRegs; ++k) {
      mk[k] = -INFINITY;
      lk[k] = 0.f;
#pragma unroll
      for (int v = 0; v < V; ++v) ok[k][v] = 0.f;
      if (k < ntot) {
        const int64_t r = row_of(k);
        mk[k] = p.part_ml[r * 2];
        lk[k] = p.part_ml[r * 2 + 1];
        const float* po = p.part_o + r * D + lane * V;
        if constexpr (V == 4) {
          const float4 o4 = *reinterpret_cast<const float4*>(po);
          ok[k][0] = o4.x; ok[k][1] = o4.y; ok[k][2] = o4.z; ok[k][3] = o4.w;
        } else {
          const float2 o2 = *reinterpret_cast<const float2*>(po);
          ok[k][0] = o2.x; ok[k][1] = o2.y;
        }
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kCombineRegs; ++k)
      if (lk[k] > 0.f) M = fmaxf(M, mk[k]);
#pragma unroll
    for (int k = 0; k < kCombineRegs; ++k) {
      if (!(lk[k] > 0.f)) continue;  // nothing attended (or no partial k): skip, never 0 * o
      const float w = lk[k] * ex2(mk[k] - M);
#pragma unroll
      for (int v = 0; v < V; ++v) acc[v] += w * ok[k][v];
      W += w;
    }
    ntot = 0;  // done: the loops below run no iteration
  }
  float M = -INFINITY;
  for (int k = lane; k < ntot; k += 32) {
    const int64_t r = row_of(k);
    const float m = p.part_ml[r * 2];
    const float l = p.part_ml[r * 2 + 1];
    if (l > 0.f) M = fmaxf(M, m);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
#pragma unroll 4
  for (int k = 0; k < ntot; ++k) {
    const int64_t r = row_of(k);
    const float m = p.part_ml[r * 2];
    const float l = p.part_ml[r * 2 + 1];
    if (!(l > 0.f)) continue;  // nothing attended in this partial: skip it, never 0 * o
    const float w = l * ex2(m - M);
    const float* po = p.part_o + r * D + lane * V;
    if constexpr (V == 4) {
      const float4 o4 = *reinterpret_cast<const float4*>(po);
      acc[0] += w * o4.x; acc[1] += w * o4.y; acc[2] += w * o4.z; acc[3] += w * o4.w;
    } else {
      const float2 o2 = *reinterpret_cast<const float2*>(po);
      acc[0] += w * o2.x; acc[1] += w * o2.y;
    }
    W += w;
  }
  const float inv = W > 0.f ? 1.f / W : 0.f;
#pragma unroll
  for (int v = 0; v < V; ++v) {
    const float x = acc[v] * inv;
    if (p.out_dtype == PA_F32) {
      static_cast<float*>(p.out)[obase + v] = x;
    } else if (p.out_dtype == PA_BF16) {
      static_cast<__nv_bfloat16*>(p.out)[obase + v] = __float2bfloat16_rn(x);
    } else {
      static_cast<__half*>(p.out)[obase + v] = __float2half_rn(x);
    }
  }
}

// ---------------------------------------------------------------------------
// Wide form of the combine, for many partials per sequence (long sequences,
// partitions): grid (B, Hq), one CTA per (sequence, query head).  Every warp finds M with
// its lanes spread over the partials; then warp w takes partials w, w + W, ...
// (lane j weighs one of them, all lanes stream the rows over head_dim with the
// weight broadcast, the loads independent of one another), and the warps'
// sums meet in shared memory.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kCombineWarps * 32) pa_combine_wide_kernel(const DecodeParams p) {
  constexpr int V = D / 32;  // floats per lane
  __shared__ float s_acc[kCombineWarps][D];
  __shared__ float s_w[kCombineWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  const int qh = blockIdx.y;
  const int G = p.group;
  const int kvh = qh / G, h = qh - kvh * G;
  const bool live = host_plan_matches(p);
  RowParts rp{};
  if (live) rp = row_parts(p, b, h);  // the plan is complete: read it before the wait
  // the next launch on the stream may start its prologue now; it waits for
  // this grid before touching data
  griddep_launch_dependents();
  griddep_wait();  // the main kernel's partials are complete and visible
  if (!live || rp.direct || !rp.valid) return;  // written by the main kernel (or no entry)
  const int32_t nseq = (rp.s0 + rp.ns <= p.nseg_cap) ? rp.ns : 0;
  const int32_t npack = (rp.s1 + rp.np <= p.nseg_cap) ? rp.np : 0;
  const int32_t ntot = nseq + npack;
  auto row_of = [&](int32_t k) {  // partial k: own entry's first, then the pack's
    const int32_t slot = k < nseq ? rp.s0 + k : rp.s1 + (k - nseq);
    const int col = k < nseq ? rp.col0 : rp.col1;
    return part_row(p, slot, kvh, col);
  };

  float M = -INFINITY;
  for (int k = lane; k < ntot; k += 32) {
    const int64_t r = row_of(k);
    if (p.part_ml[r * 2 + 1] > 0.f) M = fmaxf(M, p.part_ml[r * 2]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));

  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;
  float W = 0.f;
  for (int r0 = 0; r0 < ntot; r0 += 32 * kCombineWarps) {
    const int k = r0 + warp + lane * kCombineWarps;  // the partial this lane weighs
    float w = 0.f;
    if (k < ntot) {
      const int64_t r = row_of(k);
      const float m = p.part_ml[r * 2];
      const float l = p.part_ml[r * 2 + 1];
      w = l > 0.f ? l * ex2(m - M) : 0.f;  // nothing attended: weight 0, row skipped
    }
    W += w;
    const int rem = ntot - r0 - warp;
    const int cnt = rem <= 0 ? 0 : min(32, (rem + kCombineWarps - 1) / kCombineWarps);
#pragma unroll 8
    for (int j = 0; j < cnt; ++j) {
      const float wj = __shfl_sync(0xffffffffu, w, j);
      const float* po = p.part_o + row_of(r0 + warp + j * kCombineWarps) * D + lane * V;
      // select, never 0 * o: a skipped row contributes nothing whatever it holds
      if constexpr (V == 4) {
        const float4 o4 = *reinterpret_cast<const float4*>(po);
        acc[0] += wj > 0.f ? wj * o4.x : 0.f;
        acc[1] += wj > 0.f ? wj * o4.y : 0.f;
        acc[2] += wj > 0.f ? wj * o4.z : 0.f;
        acc[3] += wj > 0.f ? wj * o4.w : 0.f;
      } else {
        const float2 o2 = *reinterpret_cast<const float2*>(po);
        acc[0] += wj > 0.f ? wj * o2.x : 0.f;
        acc[1] += wj > 0.f ? wj * o2.y : 0.f;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(0xffffffffu, W, o);
#pragma unroll
  for (int v = 0; v < V; ++v) s_acc[warp][lane * V + v] = acc[v];
  if (lane == 0) s_w[warp] = W;
  __syncthreads();
  if (warp != 0) return;
  float Wt = 0.f;
#pragma unroll
  for (int w2 = 0; w2 < kCombineWarps; ++w2) Wt += s_w[w2];
  const float inv = Wt > 0.f ? 1.f / Wt : 0.f;
  const int64_t obase = (static_cast<int64_t>(b) * p.num_q_heads + qh) * D + lane * V;
#pragma unroll
  for (int v = 0; v < V; ++v) {
    float x = 0.f;
#pragma unroll
    for (int w2 = 0; w2 < kCombineWarps; ++w2) x += s_acc[w2][lane * V + v];
    x *= inv;
    if (p.out_dtype == PA_F32) {
      static_cast<float*>(p.out)[obase + v] = x;
    } else if (p.out_dtype == PA_BF16) {
      static_cast<__nv_bfloat16*>(p.out)[obase + v] = __float2bfloat16_rn(x);
    } else {
      static_cast<__half*>(p.out)[obase + v] = __float2half_rn(x);
    }
  }
}

// ===========================================================================
// host side
// ===========================================================================
namespace {

using MainKernel = void (*)(const CUtensorMap, const CUtensorMap, const DecodeParams);

template <int D, int HG, int NB, int CG, bool BF, bool F8>
MainKernel main_kernel_ptr() {
  return pa_decode_main_kernel<D, HG, NB, CG, BF, F8>;
}

// Built: every (head_dim, heads per CTA) with one 8-column block per head;
// 16-bit caches also with 16 columns per warp (NB 2) and with two warps of
// 16 columns per head (NB 2, CG 2, at most 4 heads per CTA).
MainKernel select_main(int D, int HG, int NB, int CG, bool bf16, bool fp8) {
  if (fp8) {
    if (D != 128 || NB != 1 || CG != 1) return nullptr;
    switch (HG) {
      case 1: return main_kernel_ptr<128, 1, 1, 1, false, true>();
      case 2: return main_kernel_ptr<128, 2, 1, 1, false, true>();
      case 4: return main_kernel_ptr<128, 4, 1, 1, false, true>();
      case 8: return main_kernel_ptr<128, 8, 1, 1, false, true>();
      default: return nullptr;
    }
  }
#define PA_SEL(d, hg, nb, cg)                                                         \
  if (D == d && HG == hg && NB == nb && CG == cg)                                     \
    return bf16 ? main_kernel_ptr<d, hg, nb, cg, true, false>()                       \
                : main_kernel_ptr<d, hg, nb, cg, false, false>();
  PA_SEL(64, 1, 1, 1) PA_SEL(64, 2, 1, 1) PA_SEL(64, 4, 1, 1) PA_SEL(64, 8, 1, 1)
  PA_SEL(128, 1, 1, 1) PA_SEL(128, 2, 1, 1) PA_SEL(128, 4, 1, 1) PA_SEL(128, 8, 1, 1)
  PA_SEL(64, 1, 2, 1) PA_SEL(64, 2, 2, 1) PA_SEL(64, 4, 2, 1) PA_SEL(64, 8, 2, 1)
  PA_SEL(128, 1, 2, 1) PA_SEL(128, 2, 2, 1) PA_SEL(128, 4, 2, 1) PA_SEL(128, 8, 2, 1)
  PA_SEL(64, 1, 2, 2) PA_SEL(64, 2, 2, 2) PA_SEL(64, 4, 2, 2)
  PA_SEL(128, 1, 2, 2) PA_SEL(128, 2, 2, 2) PA_SEL(128, 4, 2, 2)
#undef PA_SEL
  return nullptr;
}

struct LaunchPlan {
  int HG = 0, groups = 0, stages = 0, tok_box = 0, threads = 0;
  int ctas_per_group = 0, tiles_per_part = INT_MAX, nseg_cap = 0;
  int pack_size = 1, cols = 0, nb = 1, cg = 1, q_per_entry = 0, head_dim = 0;
  int64_t rows = 0;  // output rows
  bool many_partials = false;  // long sequences / partitions: closed-form plan, wide combine
  bool umma = false;           // the tensor-memory kernel (many query columns, head_dim 128)
  UmmaKernel ukernel = nullptr;
  size_t smem = 0;
  // split (shared prompts on the tensor-memory kernel): CTAs 0 .. split_ctas-1
  // of the line run the packs on the tensor-memory kernel (grid split_ctas x
  // groups); the sequences' own tiles run on the warp-level kernel `kernel`
  // with the shape below (grid ctas_b x groups_b), as line CTAs split_ctas ..
  // ctas_per_group - 1
  bool split = false;
  int split_ctas = 0, ctas_b = 0, groups_b = 0, HG_b = 0, threads_b = 0, stages_b = 0;
  size_t smem_b = 0;
  size_t off_tiles = 0, off_segs = 0, off_start = 0, off_firstk = 0, off_meta = 0, off_ctalo = 0,
         off_pack_first = 0, off_pack_n = 0, off_pack_tiles = 0, off_seq_pack = 0,
         off_seq_pre = 0, off_ent = 0, off_o = 0, off_ml = 0, total = 0;
  MainKernel kernel = nullptr;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch shape of the warp-level main kernel for HG heads per CTA: stages of
// K and V tiles within a 200 KiB budget (at most 6), the kernel, threads,
// dynamic shared memory and resident CTAs per SM (opting into the memory).
pa_status warp_kernel_shape(int D, int HG, int NB, int CG, bool bf16, bool fp8, MainKernel* kernel,
                            int* stages, size_t* smem, int* threads, int* per_sm,
                            size_t budget = 200 * 1024) {
  const size_t tile_bytes = static_cast<size_t>(kTile) * HG * D * (fp8 ? 1 : 2);
  int ns = static_cast<int>(budget / (2 * tile_bytes));
  if (ns > 6) ns = 6;
  if (ns < 2) return PA_ERR_UNSUPPORTED;
  *stages = ns;
  *smem = 1024 + static_cast<size_t>(ns) * 2 * tile_bytes + ns * sizeof(TileInfo) +
          3 * ns * sizeof(uint64_t);
  *threads = (HG * CG + 1) * 32;
  *kernel = select_main(D, HG, NB, CG, bf16, fp8);
  if (*kernel == nullptr) return PA_ERR_UNSUPPORTED;
  const void* kfn = reinterpret_cast<const void*>(*kernel);
  if (!ensure_smem_attr(kfn, *smem)) return PA_ERR_CUDA;
  *per_sm = ctas_per_sm(kfn, *threads, *smem);
  return *per_sm >= 1 ? PA_OK : PA_ERR_CUDA;
}

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

// shared_prefix: consecutive sequences may be packed over shared leading
// blocks, min(8, 32 / group) sequences per pack, whose group-many query heads
// each take a column: 16 columns per consumer warp, two warps per KV head when
// more than 16 are needed.  Otherwise every sequence is its own entry and a
// warp holds one KV head's group columns.
// max_q_len > 0: several query tokens per sequence (num_rows query rows in
// all): entries are chunks of up to min(max_q_len, 32 / group) of them, whose
// group-many heads each take a column.
pa_status make_plan(int32_t num_seqs, int32_t Hq, int32_t Hkv, int32_t D, int32_t bs,
                    int32_t max_seq_len, int32_t partition_size, bool bf16, bool fp8,
                    bool shared_prefix, LaunchPlan* lp, int32_t max_q_len = 0,
                    int64_t num_rows = 0) {
  if (num_seqs < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || max_seq_len < 0 ||
      partition_size < 0)
    return PA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return PA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PA_ERR_UNSUPPORTED;
  if (!is_pow2(bs) || bs < 4 || bs > 256) return PA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G > 8) return PA_ERR_UNSUPPORTED;
  if (partition_size > 0 && (partition_size % kTile != 0 || partition_size % bs != 0))
    return PA_ERR_INVALID_ARG;
  int P = 1, NB = 1, CG = 1, Qc = 0;
  if (max_q_len < 0 || num_rows < 0 || num_rows > INT_MAX / 2) return PA_ERR_INVALID_ARG;
  if (max_q_len > 0) {
    if (fp8 || shared_prefix) return PA_ERR_UNSUPPORTED;
    Qc = kMaxPackCols / G < max_q_len ? kMaxPackCols / G : max_q_len;
    const int need = Qc * G;  // columns of a whole chunk
    NB = need > 8 ? 2 : 1;
    CG = (need + 8 * NB - 1) / (8 * NB);
  } else if (shared_prefix && !fp8) {
    P = kMaxPackCols / G < kMaxPack ? kMaxPackCols / G : kMaxPack;
    if (P < 2) P = 1;
    const int need = P * G;  // columns of a whole pack
    NB = need > 8 ? 2 : 1;
    CG = (need + 8 * NB - 1) / (8 * NB);
  }
  int HG = 8 / CG;
  while (Hkv % HG != 0) HG >>= 1;
  if (fp8 && D != 128) return PA_ERR_UNSUPPORTED;
  const int DCT = fp8 ? 1 : D / 64;  // 128-byte rows per (token, head) in a stage
  const int TB = bs < kTile ? bs : kTile;
  if ((HG * DCT * TB * 128) % 1024 != 0) return PA_ERR_UNSUPPORTED;
  // Entries whose query columns fill all 32 rows a KV head has in the
  // tensor-memory kernel's products (packs of 32 / G samples, chunks of
  // 32 / G query tokens), with 16-bit caches and head_dim 128, run on that
  // kernel when its shape rules also hold: four KV heads per CTA, 16-token
  // boxes (blocks of 16 tokens or more).  Narrower entries would leave rows
  // of every product idle; the warp-level kernel takes them.
  const int entry_cols = (Qc > 0 ? Qc : P) * G;
  const bool umma = (P > 1 || Qc > 0) && entry_cols >= kMaxPackCols && !fp8 && D == 128 &&
                    32 % G == 0 && TB == kTile && Hkv % 4 == 0;
  if (umma) HG = 4;
  // fp8 caches: two CTAs of four KV heads per SM (stages within 100 KiB)
  // rather than one of eight, so twice the warps hide the per-tile chain of
  // the code conversion and the MMAs (the 16-bit decode is HBM-bound and
  // keeps eight heads per CTA: 0.5% faster in a same-GPU A/B)
  size_t budget = 200 * 1024;
  if (fp8 && HG == 8) {
    HG = 4;
    budget = 100 * 1024;
  }
  lp->HG = HG;
  lp->head_dim = D;
  lp->groups = Hkv / HG;
  lp->tok_box = TB;
  lp->threads = umma ? kUmmaThreads : (HG * CG + 1) * 32;
  lp->nb = NB;
  lp->cg = CG;
  lp->umma = umma;
  const DeviceInfo* dev = current_device_info();
  if (dev == nullptr) return PA_ERR_CUDA;
  int per_sm = 0;
  if (umma) {
    int stages = 6;
    while (stages > 2 && umma_smem_bytes(stages) > static_cast<size_t>(dev->max_smem_optin))
      --stages;
    lp->stages = stages;
    lp->smem = umma_smem_bytes(stages);
    lp->ukernel = select_umma(bf16);
    if (lp->ukernel == nullptr) return PA_ERR_UNSUPPORTED;
    const void* kfn = reinterpret_cast<const void*>(lp->ukernel);
    if (!ensure_smem_attr(kfn, lp->smem)) return PA_ERR_CUDA;
    per_sm = ctas_per_sm(kfn, lp->threads, lp->smem);
    if (per_sm < 1) return PA_ERR_CUDA;
  } else {
    int threads = 0;
    const pa_status st = warp_kernel_shape(D, HG, NB, CG, bf16, fp8, &lp->kernel, &lp->stages,
                                           &lp->smem, &threads, &per_sm, budget);
    if (st != PA_OK) return st;
  }
  const int total_ctas = dev->num_sms * per_sm;
  lp->ctas_per_group = total_ctas / lp->groups > 0 ? total_ctas / lp->groups : 1;
  if (lp->ctas_per_group > kPlanMaxCtas) lp->ctas_per_group = kPlanMaxCtas;
  if (umma && P > 1) {
    // Shared prompts: the packs' prefixes on the tensor-memory kernel, every
    // sequence's own tiles (one query row: G of the 32 columns) on the
    // warp-level kernel with one column block per head, run after it.  A
    // sequence entry is short and narrow; on the tensor-memory kernel it
    // would cost a query load, an epilogue and whole products.
    int HGb = 4;
    while (Hkv % HGb != 0) HGb >>= 1;
    int per_sm_b = 0;
    const pa_status st = warp_kernel_shape(D, HGb, 1, 1, bf16, false, &lp->kernel, &lp->stages_b,
                                           &lp->smem_b, &lp->threads_b, &per_sm_b, 100 * 1024);
    if (st != PA_OK) return st;
    lp->split = true;
    lp->HG_b = HGb;
    lp->groups_b = Hkv / HGb;
    lp->ctas_b = dev->num_sms * per_sm_b / lp->groups_b;
    if (lp->ctas_b < 1) lp->ctas_b = 1;
    if (lp->ctas_per_group > kPlanMaxCtas / 2) lp->ctas_per_group = kPlanMaxCtas / 2;
    if (lp->ctas_b > kPlanMaxCtas / 2) lp->ctas_b = kPlanMaxCtas / 2;
    lp->split_ctas = lp->ctas_per_group;
    lp->ctas_per_group += lp->ctas_b;
  }

  const int64_t max_tiles = (static_cast<int64_t>(max_seq_len) + kTile - 1) / kTile;
  int64_t parts_per_seq = 1;
  if (partition_size > 0) {
    lp->tiles_per_part = partition_size / kTile;
    parts_per_seq = (max_tiles + lp->tiles_per_part - 1) / lp->tiles_per_part;
    if (parts_per_seq < 1) parts_per_seq = 1;
  }
  lp->pack_size = P;
  lp->q_per_entry = Qc;
  lp->rows = Qc > 0 ? num_rows : num_seqs;
  lp->cols = umma ? kMaxPackCols : (P > 1 || Qc > 0) ? 8 * NB * CG : G;
  // entries: at most num_seqs / 2 packs (pairs), then the sequences; or at
  // most one chunk per query row
  const int64_t max_packs = P > 1 ? num_seqs / 2 : 0;
  const int64_t entries = Qc > 0 ? num_rows : static_cast<int64_t>(num_seqs) + max_packs;
  const int64_t nseg = entries * parts_per_seq + lp->ctas_per_group;
  // partials one sequence expects: its partitions plus the CTA shares it spans
  // when the batch's work is cut evenly
  const int64_t units = Qc > 0 ? (num_rows + Qc - 1) / Qc : num_seqs;  // entries, roughly
  const int64_t expect = parts_per_seq + (lp->ctas_per_group + units - 1) /
                                             (units > 0 ? units : 1);
  lp->many_partials = expect > 6;
  if (nseg > INT_MAX / 2) return PA_ERR_UNSUPPORTED;
  lp->nseg_cap = static_cast<int>(nseg);
  auto words = [](int64_t n) { return align_up(static_cast<size_t>(n) * 4, 256); };
  lp->off_tiles = 0;
  lp->off_segs = lp->off_tiles + words(entries + 1);
  lp->off_start = lp->off_segs + words(entries + 1);
  lp->off_firstk = lp->off_start + words(lp->ctas_per_group);
  lp->off_ctalo = lp->off_firstk + words(lp->ctas_per_group);
  lp->off_meta = lp->off_ctalo + words(lp->ctas_per_group + 1);
  size_t off = lp->off_meta + words(2);
  if (lp->pack_size > 1) {
    lp->off_pack_first = off;
    lp->off_pack_n = lp->off_pack_first + words(max_packs + 1);
    lp->off_pack_tiles = lp->off_pack_n + words(max_packs + 1);
    lp->off_seq_pack = lp->off_pack_tiles + words(max_packs + 1);
    lp->off_seq_pre = lp->off_seq_pack + words(num_seqs);
    off = lp->off_seq_pre + words(num_seqs);
  }
  if (Qc > 0) {  // ent_b, ent_q0, ent_nq, ent_tok, q_entry: one row each
    lp->off_ent = off;
    off = lp->off_ent + 5 * words(num_rows);
  }
  lp->off_o = off;
  const size_t o_bytes = static_cast<size_t>(Hkv) * nseg * lp->cols * D * sizeof(float);
  lp->off_ml = lp->off_o + align_up(o_bytes, 256);
  const size_t ml_bytes = static_cast<size_t>(Hkv) * nseg * lp->cols * 2 * sizeof(float);
  lp->total = lp->off_ml + align_up(ml_bytes, 256);
  return PA_OK;
}

}  // namespace
}  // namespace pa

using namespace pa;

namespace {

// The larger of the 16-bit and the fp8-cache plans of one shape.
pa_status workspace_bytes(int32_t num_seqs, int32_t Hq, int32_t Hkv, int32_t D, int32_t bs,
                          int32_t max_seq_len, int32_t partition_size, bool shared_prefix,
                          size_t* bytes, int32_t max_q_len = 0, int64_t num_rows = 0) {
  LaunchPlan lp;
  const pa_status st = make_plan(num_seqs, Hq, Hkv, D, bs, max_seq_len, partition_size, true,
                                 false, shared_prefix, &lp, max_q_len, num_rows);
  if (st != PA_OK) return st;
  *bytes = lp.total;
  LaunchPlan lp8;
  if (max_q_len == 0 &&
      make_plan(num_seqs, Hq, Hkv, D, bs, max_seq_len, partition_size, false, true,
                shared_prefix, &lp8) == PA_OK &&
      lp8.total > *bytes)
    *bytes = lp8.total;
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                               int32_t num_kv_heads, int32_t head_dim,
                                               int32_t block_size, int32_t max_seq_len,
                                               int32_t partition_size, size_t* bytes) {
  if (bytes == nullptr) return PA_ERR_INVALID_ARG;
  return workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                         max_seq_len, partition_size, false, bytes);
}

extern "C" pa_status pa_decode_multi_query_workspace_bytes(
    int32_t num_seqs, int32_t num_query_rows, int32_t max_q_len, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t max_seq_len,
    int32_t partition_size, size_t* bytes) {
  if (bytes == nullptr || max_q_len <= 0 || num_query_rows < 0) return PA_ERR_INVALID_ARG;
  return workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                         max_seq_len, partition_size, false, bytes, max_q_len, num_query_rows);
}

extern "C" pa_status pa_decode_shared_prefix_workspace_bytes(
    int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t max_seq_len, int32_t partition_size, size_t* bytes) {
  if (bytes == nullptr) return PA_ERR_INVALID_ARG;
  return workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                         max_seq_len, partition_size, true, bytes);
}

namespace {

std::atomic<uint64_t> g_consumer_wait_ns{kWaitLimitNs};

}  // namespace

uint64_t pa::consumer_wait_limit_ns() {
  return g_consumer_wait_ns.load(std::memory_order_relaxed);
}

extern "C" void pa_set_consumer_wait_limit_ns(uint64_t ns) {
  g_consumer_wait_ns.store(ns == 0 ? kWaitLimitNs : ns, std::memory_order_relaxed);
}

namespace {

// Everything one decode call launches with: the launch shape, the kernel
// parameters and the K/V tensor maps.
struct DecodeSetup {
  LaunchPlan lp;
  DecodeParams p;
  CUtensorMap tmK, tmV;
  CUtensorMap tmQ;  // the tensor-memory kernel's query rows
  CUtensorMap tmK_b, tmV_b;  // split: the warp-level kernel's K/V maps (mode_b)
  int mode_b = 0;
};

// Shared by the 16-bit and the fp8 entry points: validates the arguments,
// chooses the launch shape and fills *su.  Returns PA_OK with su->p.num_seqs
// == 0 when there is nothing to do.  elem_bytes is 1 for E4M3 codes; then
// q_dtype is the query's type and k_scale / v_scale are set.
pa_status setup_decode(void* out, pa_dtype out_dtype, const void* query, pa_dtype q_dtype,
                       const void* key_cache, const void* value_cache, int elem_bytes,
                       const float* k_scale, const float* v_scale,
                       const int32_t* block_tables, int32_t block_table_stride,
                       const int32_t* seq_lens, int32_t num_seqs, int32_t max_seq_len,
                       int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                       int32_t num_blocks, int32_t block_size, float scale,
                       int32_t partition_size, const int32_t* shared_blocks, void* workspace,
                       size_t workspace_bytes, int32_t* device_error_flag, DecodeSetup* su,
                       const pa_cache_strides* cache_strides = nullptr,
                       const int32_t* q_start = nullptr, int32_t num_rows = 0,
                       int32_t max_q_len = 0) {
  std::memset(&su->p, 0, sizeof(su->p));
  if (num_seqs < 0 || num_rows < 0) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || (q_start != nullptr && num_rows == 0)) return PA_OK;
  if (q_start != nullptr && (max_q_len <= 0 || !aligned(q_start, 4))) return PA_ERR_INVALID_ARG;
  if (!out || !query || !key_cache || !value_cache || !block_tables || !seq_lens || !workspace)
    return PA_ERR_INVALID_ARG;
  const bool fp8 = elem_bytes == 1;
  if (fp8 && (!k_scale || !v_scale || !aligned(k_scale, 4) || !aligned(v_scale, 4)))
    return PA_ERR_INVALID_ARG;
  if (q_dtype != PA_F16 && q_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (out_dtype != PA_F16 && out_dtype != PA_BF16 && out_dtype != PA_F32)
    return PA_ERR_INVALID_ARG;
  if (num_blocks <= 0 || !(scale == scale)) return PA_ERR_INVALID_ARG;
  LaunchPlan& lp = su->lp;
  lp = LaunchPlan();
  if (shared_blocks != nullptr && !aligned(shared_blocks, 4)) return PA_ERR_INVALID_ARG;
  pa_status st = make_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                           max_seq_len, partition_size, !fp8 && q_dtype == PA_BF16, fp8,
                           shared_blocks != nullptr, &lp, q_start != nullptr ? max_q_len : 0,
                           num_rows);
  if (st != PA_OK) return st;
  const int64_t need_blocks = (static_cast<int64_t>(max_seq_len) + block_size - 1) / block_size;
  if (block_table_stride < need_blocks) return PA_ERR_INVALID_ARG;
  if (workspace_bytes < lp.total) return PA_ERR_INVALID_ARG;
  if (!aligned(key_cache, 16) || !aligned(value_cache, 16) || !aligned(query, 16) ||
      !aligned(workspace, 256) || !aligned(out, out_dtype == PA_F32 ? 4 : 2) ||
      !aligned(block_tables, 4) || !aligned(seq_lens, 4))
    return PA_ERR_INVALID_ARG;

  const int HG = lp.HG, D = head_dim;
  const uint64_t e = static_cast<uint64_t>(elem_bytes);
  // pool strides in bytes (token, head, block); head_dim elements contiguous
  uint64_t tok_b = static_cast<uint64_t>(num_kv_heads) * D * e, head_b = D * e,
           blk_b = static_cast<uint64_t>(block_size) * num_kv_heads * D * e;
  if (cache_strides != nullptr) {
    if (cache_strides->block_stride <= 0 || cache_strides->token_stride <= 0 ||
        cache_strides->head_stride <= 0)
      return PA_ERR_INVALID_ARG;
    tok_b = static_cast<uint64_t>(cache_strides->token_stride) * e;
    head_b = static_cast<uint64_t>(cache_strides->head_stride) * e;
    blk_b = static_cast<uint64_t>(cache_strides->block_stride) * e;
    if (tok_b % 16 != 0 || head_b % 16 != 0 || blk_b % 16 != 0) return PA_ERR_INVALID_ARG;
  }
  const int DCT = fp8 ? 1 : D / 64;           // 128-byte rows per (token, head)
  const uint32_t inner = fp8 ? 128u : 64u;    // elements in one 128-byte row
  // The warp-level kernel's maps for HGx heads per CTA.  mode 0: dims {row,
  // tokens, d-chunks, heads, blocks}, box {row, TB, DCT, HGx, 1}; mode 1 (when
  // the driver rejects mode 0): dims {row, d-chunks, heads, tokens, blocks},
  // box {row, 1, 1, TB, 1}.
  auto warp_maps = [&](int HGx, CUtensorMap* mk, CUtensorMap* mv, int* m) {
    const uint64_t dims0[5] = {inner, (uint64_t)block_size, (uint64_t)DCT,
                               (uint64_t)num_kv_heads, (uint64_t)num_blocks};
    const uint64_t str0[4] = {tok_b, 128, head_b, blk_b};
    const uint32_t box0[5] = {inner, (uint32_t)lp.tok_box, (uint32_t)DCT, (uint32_t)HGx, 1};
    const uint64_t dims1[5] = {inner, (uint64_t)DCT, (uint64_t)num_kv_heads,
                               (uint64_t)block_size, (uint64_t)num_blocks};
    const uint64_t str1[4] = {128, head_b, tok_b, blk_b};
    const uint32_t box1[5] = {inner, 1, 1, (uint32_t)lp.tok_box, 1};
    if (get_tensor_map(mk, key_cache, dims0, str0, box0, elem_bytes) &&
        get_tensor_map(mv, value_cache, dims0, str0, box0, elem_bytes)) {
      *m = 0;
      return true;
    }
    if (lp.tok_box * 128 % 1024 == 0 &&
        get_tensor_map(mk, key_cache, dims1, str1, box1, elem_bytes) &&
        get_tensor_map(mv, value_cache, dims1, str1, box1, elem_bytes)) {
      *m = 1;
      return true;
    }
    return false;
  };
  int mode = 0;
  if (lp.split && !warp_maps(lp.HG_b, &su->tmK_b, &su->tmV_b, &su->mode_b))
    return PA_ERR_UNSUPPORTED;
  if (lp.umma) {
    // mode 2: dims {row, tokens, heads, d-chunks, blocks}, box {row, 16, HG, 2, 1}:
    // the rows of one d-chunk of all HG heads are contiguous in the stage
    const uint64_t dims2[5] = {inner, (uint64_t)block_size, (uint64_t)num_kv_heads,
                               (uint64_t)DCT, (uint64_t)num_blocks};
    const uint64_t str2[4] = {tok_b, head_b, 128, blk_b};
    const uint32_t box2[5] = {inner, (uint32_t)lp.tok_box, (uint32_t)HG, (uint32_t)DCT, 1};
    if (!get_tensor_map(&su->tmK, key_cache, dims2, str2, box2, elem_bytes) ||
        !get_tensor_map(&su->tmV, value_cache, dims2, str2, box2, elem_bytes))
      return PA_ERR_UNSUPPORTED;
    mode = 2;
  } else if (!warp_maps(HG, &su->tmK, &su->tmV, &mode)) {
    return PA_ERR_UNSUPPORTED;
  }
  if (lp.umma) {
    // query rows [rows][Hq][D] as {64 elements, 2 d-chunks, Hq, rows}; a box
    // is 64 elements of G heads of 32 / G rows: 32 rows of 128 bytes
    const int G = num_q_heads / num_kv_heads;
    const uint64_t qd[5] = {64, 2, (uint64_t)num_q_heads, (uint64_t)lp.rows, 1};
    const uint64_t qs[4] = {128, 256, (uint64_t)num_q_heads * 256,
                            (uint64_t)lp.rows * num_q_heads * 256};
    const uint32_t qb[5] = {64, 1, (uint32_t)G, (uint32_t)(32 / G), 1};
    if (!get_tensor_map(&su->tmQ, query, qd, qs, qb, 2, 4)) return PA_ERR_UNSUPPORTED;
  }

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeParams& p = su->p;
  p.out = out;
  p.query = static_cast<const uint16_t*>(query);
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.table_stride = block_table_stride;
  p.out_dtype = out_dtype;
  p.num_seqs = num_seqs;
  p.num_rows = static_cast<int32_t>(lp.rows);
  p.max_seq_len = max_seq_len;
  p.num_q_heads = num_q_heads;
  p.group = num_q_heads / num_kv_heads;
  p.num_kv_heads = num_kv_heads;
  p.num_blocks = num_blocks;
  p.block_size = block_size;
  p.tiles_per_part = lp.tiles_per_part;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.ctas_per_group = lp.ctas_per_group;
  p.split_ctas = lp.split ? lp.split_ctas : 0;
  p.cta_base = 0;
  p.heads_per_cta = HG;
  p.nseg_cap = lp.nseg_cap;
  p.stages = lp.stages;
  p.tok_box = lp.tok_box;
  p.tma_mode = mode;
  p.plan_closed = lp.many_partials ? 1 : 0;
  p.plan_tiles = reinterpret_cast<int32_t*>(ws + lp.off_tiles);
  p.seg_base = reinterpret_cast<int32_t*>(ws + lp.off_segs);
  p.start_seq = reinterpret_cast<int32_t*>(ws + lp.off_start);
  p.first_k = reinterpret_cast<int32_t*>(ws + lp.off_firstk);
  p.cta_lo = reinterpret_cast<int32_t*>(ws + lp.off_ctalo);
  p.meta = reinterpret_cast<int32_t*>(ws + lp.off_meta);
  if (q_start != nullptr) {
    p.q_start = q_start;
    p.q_per_entry = lp.q_per_entry;
    const size_t w = align_up(static_cast<size_t>(lp.rows) * 4, 256);
    p.ent_b = reinterpret_cast<int32_t*>(ws + lp.off_ent);
    p.ent_q0 = reinterpret_cast<int32_t*>(ws + lp.off_ent + w);
    p.ent_nq = reinterpret_cast<int32_t*>(ws + lp.off_ent + 2 * w);
    p.ent_tok = reinterpret_cast<int32_t*>(ws + lp.off_ent + 3 * w);
    p.q_entry = reinterpret_cast<int32_t*>(ws + lp.off_ent + 4 * w);
  }
  p.shared_blocks = shared_blocks;
  p.pack_size = lp.pack_size;
  p.cols = lp.cols;
  if (lp.pack_size > 1) {
    p.pack_first = reinterpret_cast<int32_t*>(ws + lp.off_pack_first);
    p.pack_n = reinterpret_cast<int32_t*>(ws + lp.off_pack_n);
    p.pack_tiles = reinterpret_cast<int32_t*>(ws + lp.off_pack_tiles);
    p.seq_pack = reinterpret_cast<int32_t*>(ws + lp.off_seq_pack);
    p.seq_pre = reinterpret_cast<int32_t*>(ws + lp.off_seq_pre);
  }
  p.part_o = reinterpret_cast<float*>(ws + lp.off_o);
  p.part_ml = reinterpret_cast<float*>(ws + lp.off_ml);
  p.err = device_error_flag;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.q_bf16 = q_dtype == PA_BF16 ? 1 : 0;
  p.out_vec16 = aligned(out, 16) ? 1 : 0;
  p.consumer_wait_ns = consumer_wait_limit_ns();
  return PA_OK;
}

// Launches a prepared call on `s`: the plan kernel (unless the plan was
// computed on the host, su.p.host_plan set), the main kernel and, when some
// output row has partials to merge, the combine.  All launches use
// programmatic dependent launch: each may start while its predecessor runs and
// waits (griddepcontrol.wait) before touching data.
pa_status launch_setup(const DecodeSetup& su, cudaStream_t s, bool run_combine = true) {
  const LaunchPlan& lp = su.lp;
  const DecodeParams& p = su.p;
  if (p.host_plan == nullptr &&
      PdlLaunch(s, dim3(1), dim3(kPlanThreads))(pa_plan_kernel, p) != cudaSuccess)
    return PA_ERR_CUDA;
  const int ctas_a = lp.split ? lp.split_ctas : lp.ctas_per_group;
  PdlLaunch main_launch(s, dim3(ctas_a, lp.groups), dim3(lp.threads), lp.smem);
  const cudaError_t e2 = lp.umma ? main_launch(lp.ukernel, su.tmK, su.tmV, su.tmQ, p)
                                 : main_launch(lp.kernel, su.tmK, su.tmV, p);
  if (e2 != cudaSuccess) return PA_ERR_CUDA;
  if (lp.split) {  // the sequences' own tiles: line CTAs split_ctas .. ctas_per_group - 1
    DecodeParams pb = p;
    pb.cta_base = lp.split_ctas;
    pb.heads_per_cta = lp.HG_b;
    pb.stages = lp.stages_b;
    pb.tma_mode = su.mode_b;
    PdlLaunch seq_launch(s, dim3(lp.ctas_b, lp.groups_b), dim3(lp.threads_b), lp.smem_b);
    if (seq_launch(lp.kernel, su.tmK_b, su.tmV_b, pb) != cudaSuccess) return PA_ERR_CUDA;
  }
  if (!run_combine) return PA_OK;
  const int D = lp.head_dim;
  cudaError_t e3;
  if (lp.many_partials) {
    PdlLaunch combine(s, dim3(static_cast<unsigned>(lp.rows), p.num_q_heads),
                      dim3(kCombineWarps * 32));
    e3 = D == 128 ? combine(pa_combine_wide_kernel<128>, p)
                  : combine(pa_combine_wide_kernel<64>, p);
  } else {
    PdlLaunch combine(s, dim3(static_cast<unsigned>(lp.rows),
                           (p.num_q_heads + kCombineWarps - 1) / kCombineWarps),
                      dim3(kCombineWarps * 32));
    e3 = D == 128 ? combine(pa_combine_narrow_kernel<128>, p)
                  : combine(pa_combine_narrow_kernel<64>, p);
  }
  return e3 == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status launch_decode(void* out, pa_dtype out_dtype, const void* query, pa_dtype q_dtype,
                        const void* key_cache, const void* value_cache, int elem_bytes,
                        const float* k_scale, const float* v_scale,
                        const int32_t* block_tables, int32_t block_table_stride,
                        const int32_t* seq_lens, int32_t num_seqs, int32_t max_seq_len,
                        int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                        int32_t num_blocks, int32_t block_size, float scale,
                        int32_t partition_size, const int32_t* shared_blocks, void* workspace,
                        size_t workspace_bytes, int32_t* device_error_flag, pa_stream_t stream,
                        const pa_cache_strides* cache_strides = nullptr,
                        const int32_t* q_start = nullptr, int32_t num_rows = 0,
                        int32_t max_q_len = 0) {
  DecodeSetup su;
  const pa_status st = setup_decode(
      out, out_dtype, query, q_dtype, key_cache, value_cache, elem_bytes, k_scale, v_scale,
      block_tables, block_table_stride, seq_lens, num_seqs, max_seq_len, num_q_heads,
      num_kv_heads, head_dim, num_blocks, block_size, scale, partition_size, shared_blocks,
      workspace, workspace_bytes, device_error_flag, &su, cache_strides, q_start, num_rows,
      max_q_len);
  if (st != PA_OK || su.p.num_seqs == 0) return st;
  return launch_setup(su, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" pa_status pa_decode_attention(
    void* out, pa_dtype out_dtype, const void* query, const void* key_cache,
    const void* value_cache, const int32_t* block_tables, int32_t block_table_stride,
    const int32_t* seq_lens, int32_t num_seqs, int32_t max_seq_len, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
    pa_dtype kv_dtype, int32_t partition_size, void* workspace, size_t workspace_bytes,
    int32_t* device_error_flag, pa_stream_t stream) {
  return launch_decode(out, out_dtype, query, kv_dtype, key_cache, value_cache, 2, nullptr,
                       nullptr, block_tables, block_table_stride, seq_lens, num_seqs,
                       max_seq_len, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size,
                       scale, partition_size, nullptr, workspace, workspace_bytes,
                       device_error_flag, stream);
}

extern "C" pa_status pa_decode_attention_fp8(
    void* out, pa_dtype out_dtype, const void* query, pa_dtype query_dtype,
    const void* key_cache, const void* value_cache, const float* k_scale, const float* v_scale,
    const int32_t* block_tables, int32_t block_table_stride, const int32_t* seq_lens,
    int32_t num_seqs, int32_t max_seq_len, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
    int32_t partition_size, void* workspace, size_t workspace_bytes,
    int32_t* device_error_flag, pa_stream_t stream) {
  return launch_decode(out, out_dtype, query, query_dtype, key_cache, value_cache, 1, k_scale,
                       v_scale, block_tables, block_table_stride, seq_lens, num_seqs,
                       max_seq_len, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size,
                       scale, partition_size, nullptr, workspace, workspace_bytes,
                       device_error_flag, stream);
}

extern "C" pa_status pa_decode_attention_strided(
    void* out, pa_dtype out_dtype, const void* query, pa_dtype query_dtype,
    const void* key_cache, const void* value_cache, const pa_cache_strides* cache_strides,
    pa_kv_cache_dtype kv_cache_dtype, const float* k_scale, const float* v_scale,
    const int32_t* block_tables, int32_t block_table_stride, const int32_t* seq_lens,
    int32_t num_seqs, int32_t max_seq_len, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
    int32_t partition_size, void* workspace, size_t workspace_bytes,
    int32_t* device_error_flag, pa_stream_t stream) {
  if (cache_strides == nullptr) return PA_ERR_INVALID_ARG;
  if (kv_cache_dtype != PA_KV_AUTO && kv_cache_dtype != PA_KV_FP8_E4M3) return PA_ERR_UNSUPPORTED;
  const bool fp8 = kv_cache_dtype == PA_KV_FP8_E4M3;
  return launch_decode(out, out_dtype, query, query_dtype, key_cache, value_cache, fp8 ? 1 : 2,
                       fp8 ? k_scale : nullptr, fp8 ? v_scale : nullptr, block_tables,
                       block_table_stride, seq_lens, num_seqs, max_seq_len, num_q_heads,
                       num_kv_heads, head_dim, num_blocks, block_size, scale, partition_size,
                       nullptr, workspace, workspace_bytes, device_error_flag, stream,
                       cache_strides);
}

extern "C" pa_status pa_decode_attention_multi_query(
    void* out, pa_dtype out_dtype, const void* query, const int32_t* q_start,
    int32_t num_query_rows, int32_t max_q_len, const void* key_cache, const void* value_cache,
    const int32_t* block_tables, int32_t block_table_stride, const int32_t* seq_lens,
    int32_t num_seqs, int32_t max_seq_len, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale, pa_dtype kv_dtype,
    int32_t partition_size, void* workspace, size_t workspace_bytes,
    int32_t* device_error_flag, pa_stream_t stream) {
  if (q_start == nullptr && num_seqs > 0) return PA_ERR_INVALID_ARG;
  return launch_decode(out, out_dtype, query, kv_dtype, key_cache, value_cache, 2, nullptr,
                       nullptr, block_tables, block_table_stride, seq_lens, num_seqs,
                       max_seq_len, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size,
                       scale, partition_size, nullptr, workspace, workspace_bytes,
                       device_error_flag, stream, nullptr, q_start, num_query_rows, max_q_len);
}

extern "C" pa_status pa_decode_attention_shared_prefix(
    void* out, pa_dtype out_dtype, const void* query, const void* key_cache,
    const void* value_cache, const int32_t* block_tables, int32_t block_table_stride,
    const int32_t* seq_lens, const int32_t* shared_blocks, int32_t num_seqs,
    int32_t max_seq_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t num_blocks, int32_t block_size, float scale, pa_dtype kv_dtype,
    int32_t partition_size, void* workspace, size_t workspace_bytes, int32_t* device_error_flag,
    pa_stream_t stream) {
  if (shared_blocks == nullptr && num_seqs > 0) return PA_ERR_INVALID_ARG;
  return launch_decode(out, out_dtype, query, kv_dtype, key_cache, value_cache, 2, nullptr,
                       nullptr, block_tables, block_table_stride, seq_lens, num_seqs,
                       max_seq_len, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size,
                       scale, partition_size, shared_blocks, workspace, workspace_bytes,
                       device_error_flag, stream);
}

// ===========================================================================
// Plans computed on the host.  The plan kernel reads the lengths on the
// device; a serving step has them on the host already, so the same
// bookkeeping can be done there and shipped with the step's other inputs,
// and the decode then starts with the main kernel.  Plain decode only (one
// query token per sequence, no packs).  Buffer layout (int32 words, 256-byte
// aligned sections): the header (kPlanHeaderWords), then tile prefix sums
// [B + 1], segment prefix sums [B + 1], start entry [C] and first segment
// index [C] of each CTA, and the first tile of each CTA's share [C + 1].
// ===========================================================================
namespace {

struct PlanOffsets {
  size_t tiles, segs, start, firstk, ctalo, total;
};

PlanOffsets plan_offsets(int64_t B, int64_t C) {
  auto words = [](int64_t n) { return align_up(static_cast<size_t>(n) * 4, 256); };
  PlanOffsets o;
  o.tiles = 256;
  o.segs = o.tiles + words(B + 1);
  o.start = o.segs + words(B + 1);
  o.firstk = o.start + words(C);
  o.ctalo = o.firstk + words(C);
  o.total = o.ctalo + words(C + 1);
  return o;
}

// The plan kernel's bookkeeping for a plain decode, by walking each
// sequence's cut points in order: the tiles of all sequences laid end to end
// (tiles[b] = tiles before sequence b), cut wherever a partition starts
// (every tpp tiles from a sequence's first tile) or a CTA's share starts
// (cta_lo[c]: the line cut evenly in virtual tiles, a sequence with tiles
// counting kEntryWeight more when B fits the plan kernel's shared prefix
// sums, as the plan kernel cuts it); seg_base[b] = segments before sequence
// b; start_seq[c], first_k[c] = the sequence holding cta_lo[c] and the index
// of the segment starting there.  Lengths are clamped to [0, max_seq_len].
// Returns false if the tile count does not fit in int32.
bool split_walk(const int32_t* lens, int32_t B, int32_t max_seq_len, int32_t tpp, int32_t C,
                int32_t* tiles, int32_t* seg_base, int32_t* start_seq, int32_t* first_k,
                int32_t* cta_lo, int32_t* total_segs, bool* split) {
  int64_t N = 0;
  for (int32_t b = 0; b < B; ++b) {
    tiles[b] = static_cast<int32_t>(N);
    const int32_t L = lens[b] < 0 ? 0 : (lens[b] > max_seq_len ? max_seq_len : lens[b]);
    N += (static_cast<int64_t>(L) + kTile - 1) / kTile;
    if (N > INT_MAX / 2) return false;
  }
  tiles[B] = static_cast<int32_t>(N);
  // the cut (the plan kernel's arithmetic): virtual starts, an even cut of
  // the virtual line, each cut mapped to its real tile
  const int64_t w = B <= kPlanSmemTiles ? kEntryWeight : 0;
  std::vector<int64_t> vs(static_cast<size_t>(B) + 1);
  int64_t nonempty = 0;
  for (int32_t b = 0; b < B; ++b) {
    vs[b] = tiles[b] + w * nonempty;
    if (tiles[b + 1] > tiles[b]) ++nonempty;
  }
  vs[B] = N + w * nonempty;
  LineCut cut;
  cut.C = C;
  cut.S = 0;
  cut.N = vs[B];
  cut.NK = 0;
  for (int32_t c = 0; c <= C; ++c) {
    const int64_t x = cut.lo(c);
    // the last entry whose virtual start is at or below x
    const int32_t e = static_cast<int32_t>(std::upper_bound(vs.begin(), vs.end(), x) - vs.begin()) - 1;
    cta_lo[c] = static_cast<int32_t>(
        e >= B ? N : entry_tile(x, vs[e], tiles[e], tiles[e + 1] - tiles[e], w));
  }
  for (int32_t c = 0; c < C; ++c) start_seq[c] = first_k[c] = 0;
  *split = false;
  int64_t seg = 0;
  for (int32_t b = 0; b < B; ++b) {
    seg_base[b] = static_cast<int32_t>(seg);
    const int64_t t0 = tiles[b], t1 = tiles[b + 1];
    if (t1 <= t0) continue;
    // first CTA whose share starts at or after t0
    int64_t c = std::lower_bound(cta_lo, cta_lo + C, static_cast<int32_t>(t0)) - cta_lo;
    int64_t part = t0;  // next partition start
    int32_t count = 0;
    int64_t last = -1;
    while (true) {
      const int64_t cta_pt = (c < C && cta_lo[c] < t1) ? cta_lo[c] : INT64_MAX;
      const int64_t part_pt = part < t1 ? part : INT64_MAX;
      if (cta_pt == INT64_MAX && part_pt == INT64_MAX) break;
      if (cta_pt <= part_pt) {
        const int32_t idx = (cta_pt == last) ? count - 1 : count;
        if (cta_pt != last) {
          ++count;
          last = cta_pt;
        }
        start_seq[c] = b;
        first_k[c] = idx;
        ++c;
      } else {
        if (part_pt != last) {
          ++count;
          last = part_pt;
        }
        part = (tpp == INT_MAX) ? INT64_MAX : part + tpp;
      }
    }
    seg += count;
    if (count > 1) *split = true;
  }
  seg_base[B] = static_cast<int32_t>(seg);
  *total_segs = static_cast<int32_t>(seg);
  return true;
}

// Writes a plan for launch shape lp into `buf` (host, plan_offsets().total
// bytes).  *needs_combine: some sequence has partials to merge.
pa_status write_plan(const LaunchPlan& lp, const int32_t* lens, int32_t B, int32_t max_seq_len,
                     uint8_t* buf, bool* needs_combine) {
  const int32_t C = lp.ctas_per_group;
  const PlanOffsets o = plan_offsets(B, C);
  int32_t* h = reinterpret_cast<int32_t*>(buf);
  for (int32_t b = 0; b < B; ++b)
    if (lens[b] < 0 || lens[b] > max_seq_len) return PA_ERR_INVALID_ARG;
  int32_t segs = 0;
  bool split = false;
  if (!split_walk(lens, B, max_seq_len, lp.tiles_per_part, C,
                  reinterpret_cast<int32_t*>(buf + o.tiles), reinterpret_cast<int32_t*>(buf + o.segs),
                  reinterpret_cast<int32_t*>(buf + o.start),
                  reinterpret_cast<int32_t*>(buf + o.firstk),
                  reinterpret_cast<int32_t*>(buf + o.ctalo), &segs, &split))
    return PA_ERR_UNSUPPORTED;
  if (segs > lp.nseg_cap) return PA_ERR_UNSUPPORTED;  // cannot happen: nseg_cap bounds it
  std::memset(h, 0, kPlanHeaderWords * sizeof(int32_t));
  h[0] = kPlanMagic;
  h[1] = B;
  h[2] = C;
  h[3] = lp.tiles_per_part;
  h[4] = reinterpret_cast<const int32_t*>(buf + o.tiles)[B];
  h[5] = segs;
  h[6] = split ? 1 : 0;
  *needs_combine = split;
  return PA_OK;
}

// Points a prepared call at a plan in device memory.
void use_device_plan(DecodeSetup* su, const void* plan) {
  const PlanOffsets o = plan_offsets(su->p.num_seqs, su->lp.ctas_per_group);
  const uint8_t* d = static_cast<const uint8_t*>(plan);
  su->p.host_plan = reinterpret_cast<const int32_t*>(d);
  su->p.plan_tiles = reinterpret_cast<int32_t*>(const_cast<uint8_t*>(d + o.tiles));
  su->p.seg_base = reinterpret_cast<int32_t*>(const_cast<uint8_t*>(d + o.segs));
  su->p.start_seq = reinterpret_cast<int32_t*>(const_cast<uint8_t*>(d + o.start));
  su->p.first_k = reinterpret_cast<int32_t*>(const_cast<uint8_t*>(d + o.firstk));
  su->p.cta_lo = reinterpret_cast<int32_t*>(const_cast<uint8_t*>(d + o.ctalo));
}

pa_status plan_shape(int32_t num_seqs, int32_t Hq, int32_t Hkv, int32_t D, int32_t bs,
                     int32_t max_seq_len, int32_t partition_size, pa_kv_cache_dtype kv,
                     LaunchPlan* lp) {
  if (kv != PA_KV_AUTO && kv != PA_KV_FP8_E4M3) return PA_ERR_UNSUPPORTED;
  if (num_seqs <= 0) return PA_ERR_INVALID_ARG;
  return make_plan(num_seqs, Hq, Hkv, D, bs, max_seq_len, partition_size, true,
                   kv == PA_KV_FP8_E4M3, false, lp);
}

}  // namespace

extern "C" pa_status pa_split_plan(const int32_t* seq_lens, int32_t num_seqs, int32_t max_seq_len,
                                   int32_t partition_size, int32_t num_ctas, int32_t* tiles,
                                   int32_t* seg_base, int32_t* start_seq, int32_t* first_k,
                                   int32_t* cta_first_tile, int32_t* num_segments,
                                   int32_t* needs_combine) {
  if (num_seqs <= 0 || max_seq_len < 0 || num_ctas <= 0 || num_ctas > kPlanMaxCtas ||
      partition_size < 0 || partition_size % kTile != 0)
    return PA_ERR_INVALID_ARG;
  if (!seq_lens || !tiles || !seg_base || !start_seq || !first_k || !cta_first_tile ||
      !num_segments || !needs_combine)
    return PA_ERR_INVALID_ARG;
  for (int32_t b = 0; b < num_seqs; ++b)
    if (seq_lens[b] < 0 || seq_lens[b] > max_seq_len) return PA_ERR_INVALID_ARG;
  const int32_t tpp = partition_size > 0 ? partition_size / kTile : INT_MAX;
  bool split = false;
  if (!split_walk(seq_lens, num_seqs, max_seq_len, tpp, num_ctas, tiles, seg_base, start_seq,
                  first_k, cta_first_tile, num_segments, &split))
    return PA_ERR_UNSUPPORTED;
  *needs_combine = split ? 1 : 0;
  return PA_OK;
}

extern "C" pa_status pa_decode_plan_bytes(int32_t num_seqs, int32_t num_q_heads,
                                          int32_t num_kv_heads, int32_t head_dim,
                                          int32_t block_size, int32_t max_seq_len,
                                          int32_t partition_size,
                                          pa_kv_cache_dtype kv_cache_dtype, size_t* bytes) {
  if (bytes == nullptr) return PA_ERR_INVALID_ARG;
  LaunchPlan lp;
  const pa_status st = plan_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                  max_seq_len, partition_size, kv_cache_dtype, &lp);
  if (st != PA_OK) return st;
  *bytes = plan_offsets(num_seqs, lp.ctas_per_group).total;
  return PA_OK;
}

extern "C" pa_status pa_decode_plan(const int32_t* seq_lens, int32_t num_seqs,
                                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t block_size, int32_t max_seq_len,
                                    int32_t partition_size, pa_kv_cache_dtype kv_cache_dtype,
                                    void* plan, size_t plan_bytes, int32_t* needs_combine) {
  if (seq_lens == nullptr || plan == nullptr || !aligned(plan, 4)) return PA_ERR_INVALID_ARG;
  LaunchPlan lp;
  pa_status st = plan_shape(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                            max_seq_len, partition_size, kv_cache_dtype, &lp);
  if (st != PA_OK) return st;
  if (plan_bytes < plan_offsets(num_seqs, lp.ctas_per_group).total) return PA_ERR_INVALID_ARG;
  bool combine = false;
  st = write_plan(lp, seq_lens, num_seqs, max_seq_len, static_cast<uint8_t*>(plan), &combine);
  if (st == PA_OK && needs_combine != nullptr) *needs_combine = combine ? 1 : 0;
  return st;
}

extern "C" pa_status pa_decode_attention_planned(
    void* out, pa_dtype out_dtype, const void* query, pa_dtype query_dtype,
    const void* key_cache, const void* value_cache, pa_kv_cache_dtype kv_cache_dtype,
    const float* k_scale, const float* v_scale, const int32_t* block_tables,
    int32_t block_table_stride, const int32_t* seq_lens, int32_t num_seqs, int32_t max_seq_len,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
    int32_t block_size, float scale, int32_t partition_size, const void* plan, void* workspace,
    size_t workspace_bytes, int32_t* device_error_flag, pa_stream_t stream) {
  if (kv_cache_dtype != PA_KV_AUTO && kv_cache_dtype != PA_KV_FP8_E4M3) return PA_ERR_UNSUPPORTED;
  if (num_seqs > 0 && (plan == nullptr || !aligned(plan, 256))) return PA_ERR_INVALID_ARG;
  const bool fp8 = kv_cache_dtype == PA_KV_FP8_E4M3;
  DecodeSetup su;
  const pa_status st = setup_decode(
      out, out_dtype, query, query_dtype, key_cache, value_cache, fp8 ? 1 : 2,
      fp8 ? k_scale : nullptr, fp8 ? v_scale : nullptr, block_tables, block_table_stride,
      seq_lens, num_seqs, max_seq_len, num_q_heads, num_kv_heads, head_dim, num_blocks,
      block_size, scale, partition_size, nullptr, workspace, workspace_bytes, device_error_flag,
      &su);
  if (st != PA_OK || su.p.num_seqs == 0) return st;
  use_device_plan(&su, plan);
  return launch_setup(su, reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// One decode step from host buffers.
// ---------------------------------------------------------------------------
namespace {

pa_status step_plan(const pa_step_shape* sh, LaunchPlan* lp) {
  if (sh == nullptr) return PA_ERR_INVALID_ARG;
  if (sh->dtype != PA_F16 && sh->dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (sh->out_dtype != PA_F16 && sh->out_dtype != PA_BF16 && sh->out_dtype != PA_F32)
    return PA_ERR_INVALID_ARG;
  if (sh->num_blocks <= 0 || sh->table_width <= 0 || sh->max_cow < 0) return PA_ERR_INVALID_ARG;
  if (sh->block_size > 0 &&
      sh->table_width < (static_cast<int64_t>(sh->max_seq_len) + sh->block_size - 1) / sh->block_size)
    return PA_ERR_INVALID_ARG;
  return plan_shape(sh->num_seqs, sh->num_q_heads, sh->num_kv_heads, sh->head_dim,
                    sh->block_size, sh->max_seq_len, sh->partition_size, sh->kv_cache_dtype, lp);
}

}  // namespace

extern "C" pa_status pa_decode_step_layout(const pa_step_shape* shape, pa_step_layout* layout) {
  if (layout == nullptr) return PA_ERR_INVALID_ARG;
  LaunchPlan lp;
  const pa_status st = step_plan(shape, &lp);
  if (st != PA_OK) return st;
  const int64_t B = shape->num_seqs, Hq = shape->num_q_heads, Hkv = shape->num_kv_heads,
                D = shape->head_dim;
  auto sec = [](int64_t bytes) { return align_up(static_cast<size_t>(bytes), 256); };
  pa_step_layout L;
  std::memset(&L, 0, sizeof(L));
  L.query = 0;
  L.new_k = L.query + sec(B * Hq * D * 2);
  L.new_v = L.new_k + sec(B * Hkv * D * 2);
  L.slot_mapping = L.new_v + sec(B * Hkv * D * 2);
  L.block_tables = L.slot_mapping + sec(B * 4);
  L.seq_lens = L.block_tables + sec(B * static_cast<int64_t>(shape->table_width) * 4);
  L.cow_pairs = L.seq_lens + sec(B * 4);
  L.plan = L.cow_pairs + sec(static_cast<int64_t>(shape->max_cow) * 8);
  L.host_bytes = L.plan + plan_offsets(B, lp.ctas_per_group).total;
  L.out_bytes = static_cast<size_t>(B * Hq * D) * (shape->out_dtype == PA_F32 ? 4 : 2);
  L.device_bytes = L.host_bytes + sec(static_cast<int64_t>(L.out_bytes)) + lp.total;
  *layout = L;
  return PA_OK;
}

namespace {

// Checks shared by the step's three parts; fills the layout.
pa_status step_check(const pa_step_shape* shape, const void* device_scratch,
                     size_t device_scratch_bytes, pa_step_layout* L) {
  if (shape == nullptr || device_scratch == nullptr) return PA_ERR_INVALID_ARG;
  const pa_status st = pa_decode_step_layout(shape, L);
  if (st != PA_OK) return st;
  if (!aligned(device_scratch, 256) || device_scratch_bytes < L->device_bytes)
    return PA_ERR_INVALID_ARG;
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_step_upload(const pa_step_shape* shape, void* host_staging,
                                           void* device_scratch, size_t device_scratch_bytes,
                                           pa_stream_t stream) {
  if (host_staging == nullptr || !aligned(host_staging, 16)) return PA_ERR_INVALID_ARG;
  pa_step_layout L;
  pa_status st = step_check(shape, device_scratch, device_scratch_bytes, &L);
  if (st != PA_OK) return st;
  LaunchPlan lp;
  st = step_plan(shape, &lp);
  if (st != PA_OK) return st;
  uint8_t* h = static_cast<uint8_t*>(host_staging);
  // the plan, from the lengths the caller wrote, goes out with the inputs
  bool combine = false;
  st = write_plan(lp, reinterpret_cast<const int32_t*>(h + L.seq_lens), shape->num_seqs,
                  shape->max_seq_len, h + L.plan, &combine);
  if (st != PA_OK) return st;
  if (cudaMemcpyAsync(device_scratch, h, L.host_bytes, cudaMemcpyHostToDevice,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PA_ERR_CUDA;
  return PA_OK;
}

extern "C" pa_status pa_decode_step_run(const pa_step_shape* shape, const void* host_staging,
                                        int32_t num_cow, void* key_cache, void* value_cache,
                                        const float* k_scale, const float* v_scale, float scale,
                                        void* device_scratch, size_t device_scratch_bytes,
                                        int32_t* device_error_flag, pa_stream_t stream) {
  if (!host_staging || !key_cache || !value_cache) return PA_ERR_INVALID_ARG;
  pa_step_layout L;
  pa_status st = step_check(shape, device_scratch, device_scratch_bytes, &L);
  if (st != PA_OK) return st;
  if (num_cow < 0 || num_cow > shape->max_cow) return PA_ERR_INVALID_ARG;
  const bool fp8 = shape->kv_cache_dtype == PA_KV_FP8_E4M3;
  if (fp8 && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
  const int32_t B = shape->num_seqs, Hq = shape->num_q_heads, Hkv = shape->num_kv_heads,
                D = shape->head_dim;
  uint8_t* d = static_cast<uint8_t*>(device_scratch);
  uint8_t* d_out = d + L.host_bytes;
  uint8_t* d_ws = d_out + align_up(L.out_bytes, 256);
  const size_t ws_bytes = device_scratch_bytes - (d_ws - d);

  DecodeSetup su;
  st = setup_decode(d_out, shape->out_dtype, d + L.query, shape->dtype, key_cache, value_cache,
                    fp8 ? 1 : 2, fp8 ? k_scale : nullptr, fp8 ? v_scale : nullptr,
                    reinterpret_cast<const int32_t*>(d + L.block_tables), shape->table_width,
                    reinterpret_cast<const int32_t*>(d + L.seq_lens), B, shape->max_seq_len, Hq,
                    Hkv, D, shape->num_blocks, shape->block_size, scale, shape->partition_size,
                    nullptr, d_ws, ws_bytes, device_error_flag, &su);
  if (st != PA_OK) return st;
  // the plan pa_decode_step_upload wrote into the staging buffer (its header
  // must name this shape) is in device_scratch by the time the kernels run
  const int32_t* hdr =
      reinterpret_cast<const int32_t*>(static_cast<const uint8_t*>(host_staging) + L.plan);
  if (hdr[0] != kPlanMagic || hdr[1] != B || hdr[2] != su.lp.ctas_per_group ||
      hdr[3] != su.lp.tiles_per_part)
    return PA_ERR_INVALID_ARG;
  const bool combine = hdr[6] != 0;
  use_device_plan(&su, d + L.plan);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (num_cow > 0) {
    void* kc[1] = {key_cache};
    void* vc[1] = {value_cache};
    const int64_t block_bytes =
        static_cast<int64_t>(shape->block_size) * Hkv * D * (fp8 ? 1 : 2);
    st = pa_copy_blocks(kc, vc, 1, reinterpret_cast<const int32_t*>(d + L.cow_pairs), num_cow,
                        shape->num_blocks, block_bytes, device_error_flag, stream);
    if (st != PA_OK) return st;
  }
  const int64_t row = static_cast<int64_t>(Hkv) * D;
  st = pa_reshape_and_cache(d + L.new_k, d + L.new_v, row, row, key_cache, value_cache,
                            reinterpret_cast<const int32_t*>(d + L.slot_mapping), B,
                            shape->num_blocks, shape->block_size, Hkv, D, shape->dtype,
                            shape->kv_cache_dtype, k_scale, v_scale, device_error_flag, stream);
  if (st != PA_OK) return st;
  return launch_setup(su, s, combine);
}

extern "C" pa_status pa_decode_step_download(const pa_step_shape* shape,
                                             const void* device_scratch,
                                             size_t device_scratch_bytes, void* host_out,
                                             pa_stream_t stream) {
  if (host_out == nullptr) return PA_ERR_INVALID_ARG;
  pa_step_layout L;
  const pa_status st = step_check(shape, device_scratch, device_scratch_bytes, &L);
  if (st != PA_OK) return st;
  const uint8_t* d_out = static_cast<const uint8_t*>(device_scratch) + L.host_bytes;
  if (cudaMemcpyAsync(host_out, d_out, L.out_bytes, cudaMemcpyDeviceToHost,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PA_ERR_CUDA;
  return PA_OK;
}

extern "C" pa_status pa_decode_step(const pa_step_shape* shape, void* host_staging,
                                    int32_t num_cow, void* key_cache, void* value_cache,
                                    const float* k_scale, const float* v_scale, float scale,
                                    void* device_scratch, size_t device_scratch_bytes,
                                    void* host_out, int32_t* device_error_flag,
                                    pa_stream_t stream) {
  if (!shape || !host_staging || !key_cache || !value_cache || !device_scratch || !host_out)
    return PA_ERR_INVALID_ARG;
  // everything the later parts refuse is refused before the first copy
  if (num_cow < 0 || num_cow > shape->max_cow) return PA_ERR_INVALID_ARG;
  if (shape->kv_cache_dtype == PA_KV_FP8_E4M3 && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
  pa_status st = pa_decode_step_upload(shape, host_staging, device_scratch, device_scratch_bytes,
                                       stream);
  if (st != PA_OK) return st;
  st = pa_decode_step_run(shape, host_staging, num_cow, key_cache, value_cache, k_scale, v_scale,
                          scale, device_scratch, device_scratch_bytes, device_error_flag, stream);
  if (st != PA_OK) return st;
  return pa_decode_step_download(shape, device_scratch, device_scratch_bytes, host_out, stream);
}

// ===========================================================================
// No-allocation variant: the same launches with the workspace in a static
// device array of this file instead of caller-provided memory, for callers
// that may not allocate device memory (see pa_decode_attention_noalloc in the
// header).  In host code the array's name is only a host-side stand-in, so its
// device address is looked up once per device and passed to the kernels.
// ===========================================================================
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mu;
// Device address of g_noalloc_scratch, per device, with the id of the CUDA
// context it was looked up in: a device reset ends that context, and the next
// call (in the new context, which has a new id) looks the address up again.
void* g_noalloc_addr[64] = {};
unsigned long long g_noalloc_ctx[64] = {};

// Unique id of the calling thread's current context (0 if none or unknown).
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    looked_up = true;
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
        q1 == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
        q2 == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f1);
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(f2);
    }
  }
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Looks the array's address up on the current device the first time in each
// context; later calls in that context reuse it.
pa_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  const unsigned long long ctx = current_context_id();
  if (g_noalloc_addr[dev] == nullptr || ctx == 0 || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return PA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
    g_noalloc_ctx[dev] = current_context_id();  // the lookup made the context current
  }
  *out = g_noalloc_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_attention_noalloc(
    void* out, pa_dtype out_dtype, const void* query, const void* key_cache,
    const void* value_cache, const int32_t* block_tables, int32_t block_table_stride,
    const int32_t* seq_lens, int32_t num_seqs, int32_t max_seq_len, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks, int32_t block_size, float scale,
    pa_dtype kv_dtype, int32_t partition_size, int32_t* device_error_flag, pa_stream_t stream) {
  if (num_seqs < 0) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  size_t need = 0;
  pa_status st = pa_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                           block_size, max_seq_len, partition_size, &need);
  if (st != PA_OK) return st;
  if (need > PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_TOO_LARGE;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != PA_OK) return st;
  return pa_decode_attention(out, out_dtype, query, key_cache, value_cache, block_tables,
                             block_table_stride, seq_lens, num_seqs, max_seq_len, num_q_heads,
                             num_kv_heads, head_dim, num_blocks, block_size, scale, kv_dtype,
                             partition_size, scratch, PA_NOALLOC_SCRATCH_BYTES, device_error_flag,
                             stream);
}
