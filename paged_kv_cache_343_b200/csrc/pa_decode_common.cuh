// pa_decode_common.cuh -- what the decode kernels share: the tile record the
// producer hands to the consumers, the launch parameters, and the layout
// constants of packs, query chunks and host-computed plans.
#pragma once

#include <cuda.h>

#include <climits>
#include <cstddef>
#include <cstdint>

#include "pa_device.cuh"

namespace pa {

constexpr int kTile = 16;            // tokens per tile (MMA M of the score product)
constexpr int kPlanThreads = 256;
constexpr int kCombineWarps = 4;
constexpr int kCombineRegs = 8;  // partials a combine lane loads at once (few-partial rows)

enum : int32_t {
  kNewSeq = 1,    // first tile of a sequence in this CTA: reload Q
  kSegStart = 2,  // reset the online-softmax state
  kSegEnd = 4,    // finalise and write the segment
  kDirect = 8,    // the segment is the whole sequence: write `out` directly
  kCausal = 16,   // several query tokens of one sequence: column c sees rows <= rel + c / G
};

constexpr int kMaxPack = 8;        // sequences per pack
constexpr int kMaxPackCols = 32;   // query columns per KV head of a pack (4 blocks of 8)
constexpr int kMinPackTiles = 4;   // shared prefixes shorter than this are not packed

struct TileInfo {
  int32_t b;       // sequence (the first member of a pack)
  int32_t valid;   // tokens of this tile inside the sequence (1..16)
  int32_t mask;    // bit t set: token t takes part (valid and its block id is good)
  int32_t seg;     // segment id inside this head group
  int32_t flags;
  int32_t members;  // query rows using this tile: pack members, query tokens, or 1
  int32_t qrow0;    // query row of column 0 (column c: row qrow0 + c / G, head c % G)
  int32_t rel;      // kCausal: last visible tile row of column 0 (may be < 0 or > 15)
};

struct DecodeParams {
  void* out;
  const uint16_t* query;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  int64_t table_stride;
  int32_t out_dtype;
  int32_t num_seqs, max_seq_len, num_q_heads, num_kv_heads, group, num_blocks, block_size;
  int32_t num_rows;        // query (and output) rows: num_seqs, or the multi-query rows
  int32_t tiles_per_part;  // partition length in tiles (INT_MAX: no partitions)
  float scale_log2;        // scale * log2(e)
  int32_t ctas_per_group;  // CTAs sharing one head group's tiles (both kernels of a split)
  int32_t split_ctas;      // 0: one kernel walks the whole line; else CTAs 0 .. split_ctas-1
                           //    (the tensor-memory kernel) share the packs' tiles and the
                           //    rest (the warp-level kernel) the sequences' (LineCut)
  int32_t cta_base;        // line CTA index of this launch's blockIdx.x == 0
  int32_t heads_per_cta;   // KV heads per CTA (HG)
  int32_t nseg_cap;        // partial slots (segments)
  int32_t stages;
  int32_t tok_box;         // tokens per TMA box: min(block_size, 16)
  int32_t tma_mode;        // 0: one box per block per tile, 1: one per (head, d-half)
  int32_t plan_closed;     // 1: segment bookkeeping in closed form (many cut points per
                           //    entry); 0: walk each entry's cut points (few)
  int32_t* plan_tiles;     // [entries + 1] tile prefix sums
  int32_t* seg_base;       // [entries + 1] segment prefix sums (partial slots)
  int32_t* cta_lo;         // [ctas_per_group + 1] first tile of each CTA's share (LineCut
                           //    of the weighted line, entry_tile below); [C] = N
  int32_t* start_seq;      // [ctas_per_group] entry holding each CTA's first tile
  int32_t* first_k;        // [ctas_per_group] index of that tile's segment in its entry
  // shared prompts: packs of pack_size consecutive sequences whose block tables
  // share leading blocks are attended together over that prefix ("entries"
  // 0 .. K-1 are the packs' prefixes, K + b the rest of sequence b)
  const int32_t* shared_blocks;  // [num_seqs] leading blocks b shares with b + 1, or null
  int32_t pack_size;       // sequences per window (1: no packing)
  int32_t* pack_first;     // [num_seqs / 2] first sequence of pack k
  int32_t* pack_n;         // [num_seqs / 2] sequences of pack k (pack_size, or 2)
  int32_t* pack_tiles;     // [num_seqs / 2] prefix tiles of pack k
  int32_t* seq_pack;       // [num_seqs] pack of sequence b, or -1
  int32_t* seq_pre;        // [num_seqs] tiles of b attended through its pack
  int32_t* meta;           // [2] number of packs K (0 without packing), number of entries E
  // several query tokens per sequence ("multi-query"): entries are chunks of
  // at most q_per_entry query tokens of one sequence
  const int32_t* q_start;  // [num_seqs + 1] query rows of sequence b, or null
  int32_t q_per_entry;
  int32_t* ent_b;          // [rows] sequence of entry e
  int32_t* ent_q0;         // [rows] first query row of entry e
  int32_t* ent_nq;         // [rows] query rows of entry e
  int32_t* ent_tok;        // [rows] tokens entry e reads: one past its last query's position
  int32_t* q_entry;        // [rows] entry of query row r
  int32_t cols;            // partial columns per KV head: pack_size * group
  float* part_o;           // [nseg_cap][num_kv_heads][cols][head_dim]
  float* part_ml;          // [nseg_cap][num_kv_heads][cols][2]  (m in log2 units, l)
  int32_t* err;
  const float* k_scale;    // fp8 cache only: element = code * (*k_scale)
  const float* v_scale;
  int32_t q_bf16;          // fp8 cache only: the query is bf16 (else fp16)
  // A plan computed on the host and copied to the device (plain decode only):
  // its header, checked against this call before any work; plan_tiles,
  // seg_base, start_seq and first_k then point into the same buffer.  Null:
  // the plan kernel writes them into the workspace.
  const int32_t* host_plan;
  int32_t out_vec16;       // out is 16-byte aligned (vector stores allowed)
  uint64_t consumer_wait_ns;  // limit of the consumer warps' waits for a landed stage
};

// How the tile line of N tiles is cut into CTA shares [lo(c), lo(c + 1)).
// One kernel (S == 0): evenly over the C CTAs.  Split (0 < S < C): the
// packs' tiles [0, NK) evenly over CTAs 0 .. S-1, the sequences' tiles
// [NK, N) evenly over CTAs S .. C-1, so no share mixes the two.
struct LineCut {
  int64_t C, S, N, NK;
  __host__ __device__ int64_t lo(int64_t c) const {
    if (S == 0) return c * N / C;
    if (c < S) return c * NK / S;
    return NK + (c - S) * (N - NK) / (C - S);
  }
  // CTAs whose share starts below x, 0 <= x <= N (lo is non-decreasing in c)
  __host__ __device__ int64_t count_below(int64_t x) const {
    auto cdiv = [](int64_t a, int64_t b) { return (a + b - 1) / b; };
    if (N <= 0) return 0;
    if (S == 0) return min(C, cdiv(x * C, N));
    if (x <= NK) return NK > 0 ? min(S, cdiv(x * S, NK)) : 0;
    const int64_t C2 = C - S, N2 = N - NK;
    return S + min(C2, cdiv((x - NK) * C2, N2));
  }
};

// The cut weighs each entry switch: a CTA whose share spans several entries
// pays an epilogue, a query load and a pipeline restart per switch, so the
// line is cut evenly in virtual tiles where an entry with tiles counts its
// tiles plus kEntryWeight (its switch first).  Batches of more entries than
// the plan keeps in shared memory are cut unweighted.
constexpr int kEntryWeight = 3;  // same-GPU A/B: 3 beat 2 and 4 on longtail and multi-query

// The real tile at virtual position x of an entry that starts at virtual
// position v_e and real tile t_e and holds n_e tiles (weight w per switch):
// inside its switch the cut falls on its first tile.
__host__ __device__ __forceinline__ int64_t entry_tile(int64_t x, int64_t v_e, int64_t t_e,
                                                       int64_t n_e, int64_t w) {
  const int64_t o = x - v_e - (n_e > 0 ? w : 0);
  return t_e + (o < 0 ? 0 : (o > n_e ? n_e : o));
}

// Row of (segment, KV head, column) in the partial buffers.
__host__ __device__ __forceinline__ int64_t part_row(const DecodeParams& p, int64_t seg, int kvh,
                                                     int col) {
  return (seg * p.num_kv_heads + kvh) * p.cols + col;
}

// Limit of the consumers' waits for the next call's kernels (host side; see
// pa_set_consumer_wait_limit_ns).
uint64_t consumer_wait_limit_ns();

// Header of a host-computed plan (int32 words): magic, num_seqs, CTAs per head
// group, partition length in tiles, total tiles, total segments, whether some
// sequence has more than one segment (needs the combine).
constexpr int32_t kPlanMagic = 0x4c504150;  // "PAPL"
constexpr int kPlanHeaderWords = 8;

// True when the host plan (if any) was made for this call's shape.
__device__ __forceinline__ bool host_plan_matches(const DecodeParams& p) {
  if (p.host_plan == nullptr) return true;
  const int32_t* h = p.host_plan;
  return h[0] == kPlanMagic && h[1] == p.num_seqs && h[2] == p.ctas_per_group &&
         h[3] == p.tiles_per_part;
}

__device__ __forceinline__ int32_t clamp_len(int32_t L, int32_t max_len) {
  return L < 0 ? 0 : (L > max_len ? max_len : L);
}



// The tensor-memory kernel for entries with many query columns
// (pa_decode_umma.cu): head_dim 128, 16-bit caches, 4 KV heads per CTA,
// 16-token boxes whose rows run (d-chunk, head, token) (tma_mode 2).
using UmmaKernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                            const DecodeParams);
UmmaKernel select_umma(bool bf16);
size_t umma_smem_bytes(int stages);
constexpr int kUmmaThreads = 256;

// ---------------------------------------------------------------------------
// The members of a pack read the first member's blocks over the pack's tiles,
// so their tables must hold the same ids there; a difference is flagged
// (PA_DEVERR_BAD_SHARE).  Threads first, first + stride, ... of a warp that
// does not load tiles take the CTA's tiles [lo, hi) in turn, away from the
// producer's path.  Entries 0 .. K-1 of a line are the packs.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void check_pack_tables(const DecodeParams& p, int64_t lo, int64_t hi,
                                                  int c, int first, int stride) {
  if (p.pack_size <= 1 || p.q_start != nullptr) return;
  const int K = p.meta[0];
  int e = p.start_seq[c];
  const int bs = p.block_size;
  const int nblk = bs < kTile ? kTile / bs : 1;  // blocks a tile reads
  for (int64_t t = lo + first; t < hi && e < K; t += stride) {
    while (e < K && t >= p.plan_tiles[e + 1]) ++e;
    if (e >= K) break;
    const int64_t ti = t - p.plan_tiles[e];  // tile of the pack's prefix
    const int members = p.pack_n[e];
    const int32_t* row = p.block_tables + static_cast<int64_t>(p.pack_first[e]) * p.table_stride;
    const int64_t idx0 = bs < kTile ? ti * nblk : ti * kTile / bs;
    for (int kk = 0; kk < nblk; ++kk) {
      const int32_t id = __ldg(row + idx0 + kk);
#pragma unroll
      for (int m = 1; m < kMaxPack; ++m)
        if (m < members && __ldg(row + static_cast<int64_t>(m) * p.table_stride + idx0 + kk) != id)
          flag_error(p.err, PA_DEVERR_BAD_SHARE);
    }
  }
}

// ---------------------------------------------------------------------------
// The producer warp's loop (one elected lane), shared by the decode kernels:
// walks the CTA's tiles [lo, hi) of the tile line entry by entry, looks up
// each tile's block ids (one table lookup per block), loads its K and V with
// TMA into the stage ring (full_k / full_v of stage s at full_k0 + 8 s ...;
// a stage is reused once empty[s] completes), and publishes each tile's
// TileInfo.  on_entry(n, qrow0) runs after the first tile of the CTA's n-th
// entry has been published (n = 0, 1, ...); returning false stops the loop.
// Finally waits (bounded) for its own copies in flight.
// ---------------------------------------------------------------------------
template <int HG, int DCT, class OnEntry>
__device__ __forceinline__ void produce_tiles(const DecodeParams& p, const CUtensorMap* tmK,
                                              const CUtensorMap* tmV, uint32_t smem_base,
                                              uint32_t kTileBytes, TileInfo* info,
                                              uint32_t full_k0, uint32_t full_v0, uint32_t empty0,
                                              int NS, int64_t lo, int64_t hi, int c, int hg,
                                              bool plain, OnEntry on_entry) {
  auto full_k = [&](int s) { return full_k0 + 8u * s; };
  auto full_v = [&](int s) { return full_v0 + 8u * s; };
  auto empty = [&](int s) { return empty0 + 8u * s; };
  int32_t n_entry = 0;
  const uint64_t policy = l2_policy_evict_first();
  const int bs = p.block_size;
  const int TB = p.tok_box;
  const uint32_t box_bytes = static_cast<uint32_t>(HG * DCT * TB * 128);
  const int bpt = bs < kTile ? kTile / bs : 1;  // blocks per tile
  const int K = plain ? 0 : p.meta[0];
  // the entry being walked: tiles t_first .. t_first + n_e - 1 of the line,
  // which are tiles i0 .. i0 + n_e - 1 of sequence b (of every pack member)
  int e = p.start_seq[c];
  int b = 0, members = 1;
  int32_t t_first = 0, n_e = 0, i0 = 0, L_b = 0, seg_e = 0, nseg_e = 0;
  int32_t qrow0 = 0, lim0 = 0;  // first query row; causal: position of query 0
  bool pack = false;
  bool stale = false;  // the entry's tile count disagrees with its length
  const int32_t* row = p.block_tables;
  auto enter = [&](int ent) {
    t_first = p.plan_tiles[ent];
    n_e = p.plan_tiles[ent + 1] - t_first;
    seg_e = p.seg_base[ent];
    nseg_e = p.seg_base[ent + 1] - seg_e;
    pack = false;
    if (p.q_start != nullptr) {
      b = p.ent_b[ent];
      members = p.ent_nq[ent];
      i0 = 0;
      L_b = p.ent_tok[ent];
      qrow0 = p.ent_q0[ent];
      lim0 = L_b - members;
    } else if (ent < K) {
      b = p.pack_first[ent];
      members = p.pack_n[ent];
      i0 = 0;
      L_b = n_e * kTile;
      qrow0 = b;
      pack = true;
    } else {
      b = ent - K;
      members = 1;
      i0 = p.pack_size > 1 ? p.seq_pre[b] : 0;
      L_b = clamp_len(p.seq_lens[b], p.max_seq_len);
      qrow0 = b;
    }
    // A plan made on the host from other lengths: its tiles of this entry
    // are attended as empty (no table entry or pool row is read).
    stale = plain && (L_b + kTile - 1) / kTile != n_e;
    if (stale) flag_error(p.err, PA_DEVERR_BAD_SEQLEN);
    row = p.block_tables + static_cast<int64_t>(b) * p.table_stride;
  };
  enter(e);
  int32_t k = p.first_k[c] - 1;  // segment index inside the entry (advanced at starts)
  int32_t i = static_cast<int32_t>(lo - t_first);
  bool new_seq = true;
  int stage = 0;
  uint32_t phase = 0;
  int64_t issued = 0;
  // blocks longer than a tile: the id of the block the last tile read, so a
  // block's tiles after its first reuse it (one table lookup per block)
  const int32_t* id_row = nullptr;
  int64_t id_idx = -1;
  int32_t id_val = -1;
  // Tile index inside its partition: segments start at the CTA's first
  // tile, at an entry's first tile and at every partition start, and end
  // before the next start or at the CTA's last tile.
  const int32_t tpp = p.tiles_per_part;
  int32_t ip = tpp == INT_MAX ? i : i % tpp;
  for (int64_t t = lo; t < hi; ++t, ++i) {
    while (i >= n_e) {  // next entry that has tiles
      enter(++e);
      k = -1;
      i = 0;
      ip = 0;
      new_seq = true;
    }
    const int32_t ti_seq = i0 + i;  // tile index inside the sequence
    const int32_t valid = stale ? 0 : min(kTile, L_b - ti_seq * kTile);
    int32_t flags = new_seq ? kNewSeq : 0;
    if (t == lo || ip == 0) {
      flags |= kSegStart;
      ++k;
    }
    if (t == hi - 1 || i == n_e - 1 || ip == tpp - 1) flags |= kSegEnd;
    // one segment holds the whole attention of every query row of the entry
    if (nseg_e == 1 && !pack && i0 == 0) flags |= kDirect;
    if (p.q_start != nullptr) flags |= kCausal;
    new_seq = false;
    if (++ip == tpp) ip = 0;
    uint32_t mask = valid >= kTile ? 0xffffu : ((1u << valid) - 1u);
    // the first block id is loaded before the wait for a free stage
    const int64_t idx0 = bs <= kTile ? static_cast<int64_t>(ti_seq) * bpt
                                     : static_cast<int64_t>(ti_seq) * kTile / bs;
    int32_t id0 = -1;
    if (!stale) {
      if (bs > kTile && row == id_row && idx0 == id_idx) {
        id0 = id_val;
      } else {
        id0 = __ldg(row + idx0);
        id_row = row;
        id_idx = idx0;
        id_val = id0;
      }
    }

    if (!mbar_wait(empty(stage), phase ^ 1u, p.err)) break;
    const uint32_t kdst = smem_base + static_cast<uint32_t>(stage) * 2u * kTileBytes;
    const uint32_t vdst = kdst + kTileBytes;
    // one box per block of the tile; each copy's bytes are announced on the
    // stage's barriers just before it is issued
    auto issue = [&](uint32_t off, int32_t tok_off, int32_t id) {
      mbar_expect_tx(full_k(stage), box_bytes);
      mbar_expect_tx(full_v(stage), box_bytes);
      if (p.tma_mode == 0) {
        tma_load_5d(kdst + off, tmK, full_k(stage), 0, tok_off, 0, hg * HG, id, policy);
        tma_load_5d(vdst + off, tmV, full_v(stage), 0, tok_off, 0, hg * HG, id, policy);
      } else if (p.tma_mode == 2) {  // dims {row, tokens, heads, d-chunks, blocks}
        tma_load_5d(kdst + off, tmK, full_k(stage), 0, tok_off, hg * HG, 0, id, policy);
        tma_load_5d(vdst + off, tmV, full_v(stage), 0, tok_off, hg * HG, 0, id, policy);
      } else {
        for (int hh = 0; hh < HG; ++hh) {
          for (int dc = 0; dc < DCT; ++dc) {
            const uint32_t o2 = off + ((hh * DCT + dc) * TB) * 128u;
            tma_load_5d(kdst + o2, tmK, full_k(stage), 0, dc, hg * HG + hh, tok_off, id,
                        policy);
            tma_load_5d(vdst + o2, tmV, full_v(stage), 0, dc, hg * HG + hh, tok_off, id,
                        policy);
          }
        }
      }
    };
    if (bs <= kTile) {
#pragma unroll
      for (int kk = 0; kk < kTile / 4; ++kk) {
        const int tok0 = kk * bs;
        if (kk < bpt && tok0 < valid) {
          const int32_t id = kk == 0 ? id0 : __ldg(row + idx0 + kk);
          if (id < 0 || id >= p.num_blocks) {
            flag_error(p.err, PA_DEVERR_BAD_BLOCK);
            mask &= ~(((1u << bs) - 1u) << tok0);
          } else {
            issue(static_cast<uint32_t>(kk) * box_bytes, 0, id);
          }
        }
      }
    } else if (!stale) {
      if (id0 < 0 || id0 >= p.num_blocks) {
        flag_error(p.err, PA_DEVERR_BAD_BLOCK);
        mask = 0;
      } else {
        issue(0, static_cast<int32_t>((static_cast<int64_t>(ti_seq) * kTile) % bs), id0);
      }
    }
    TileInfo& ti = info[stage];
    ti.b = b;
    ti.valid = valid;
    ti.mask = static_cast<int32_t>(mask);
    ti.seg = seg_e + k;
    ti.flags = flags;
    ti.members = members;
    ti.qrow0 = qrow0;
    ti.rel = (flags & kCausal) ? lim0 - ti_seq * kTile : kTile;  // kTile: every row visible
    // the one arrival of the phase: it completes once the announced bytes land
    mbar_arrive(full_k(stage));
    mbar_arrive(full_v(stage));
    ++issued;
    if (++stage == NS) { stage = 0; phase ^= 1u; }
    if ((flags & kNewSeq) && !on_entry(n_entry++, qrow0)) break;
  }
  // Wait (bounded) until every load this warp issued has landed, so that no
  // copy is in flight into shared memory when the CTA retires.
  for (int64_t k = (issued > NS ? issued - NS : 0); k < issued; ++k) {
    const int s = static_cast<int>(k % NS);
    const uint32_t par = static_cast<uint32_t>((k / NS) & 1);
    if (!mbar_wait(full_k(s), par, p.err)) break;
    if (!mbar_wait(full_v(s), par, p.err)) break;
  }
}

}  // namespace pa
