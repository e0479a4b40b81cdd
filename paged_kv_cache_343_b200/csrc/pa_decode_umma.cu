// pa_decode_umma.cu -- the decode main kernel on the fifth-generation tensor
// cores (tcgen05, tensor memory), for entries with many query columns: packs
// of samples over a shared prompt ("PagedAttention", "Sharing and
// copy-on-write": the samples' tables point at the same prompt blocks, so a
// block read once serves every sample's query) and chunks of several query
// tokens of one sequence.  Same plan, tile line, segments, partials and
// combine as the warp-level kernel of pa_decode.cu; only the consumer side
// differs.
//
// A CTA takes four KV heads.  Rows of every product are the 128 pairs
// (head h, query column c) of the entry (c < 32: pack member or query token
// times the group's query heads), so every tensor-memory lane holds one row.
// Per 16-token tile:
//   S = Q . K^T        eight 128 x 64 x 16 MMAs: the columns are the 64 pairs
//                      (KV head g, token t) of the tile, read in place from
//                      the stage; only the blocks h = g are used;
//   softmax            the thread owning row (h, c) reads its 16 scores from
//                      tensor memory: no cross-thread reduction; the running
//                      maximum moves only when a tile's maximum exceeds it by
//                      2^8, so the accumulator is rarely rescaled;
//   O += P . V         P goes back to tensor memory as two 16-bit halves (hi,
//                      lo), block diagonal: row (h, c) holds its 16 weights in
//                      the columns of head h and zeros elsewhere (written
//                      once), so eight 128 x 128 x 16 MMAs (four heads x two
//                      halves) read P from tensor memory and each head's V in
//                      place, and every row gathers only its own head's V.
// One thread issues a tcgen05.mma about every 60 cycles, so few large MMAs
// matter more than their size, and the S products (warp 5) and the P.V
// products (warp 6) have an issuing thread each, running ahead of and behind
// the softmax.  Warps 0..3: softmax and epilogue of heads 0..3 (tensor-memory
// sub-partition = warp), 4: producer (TMA: K/V tiles and each entry's query
// rows), 5: S issuer and tensor-memory owner, 6: P.V issuer, 7: checks that
// a pack's members share the blocks read for them.  Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>

#include "pa_decode_common.cuh"
#include "pa_device.cuh"
#include "pa_umma.cuh"

namespace pa {

namespace {

constexpr int kUD = 128;                     // head_dim of this kernel
constexpr int kUH = 4;                       // KV heads per CTA
constexpr int kUThreads = kUmmaThreads;      // 8 warps
constexpr float kLazyLog2 = 8.0f;            // growth of a row maximum that forces a rescale
constexpr uint32_t kUTileBytes = kTile * kUH * kUD * 2;  // K (or V) of one tile: 16 KiB
constexpr uint32_t kUQBytes = 2 * 128 * 128;             // query rows of an entry: 32 KiB
constexpr int kUQBufs = 2;                               // query buffers (entries in flight)
// tensor-memory columns: O [0, 128), three S buffers [128, 320), three P
// buffers of two halves [320, 512)
constexpr int kUBufs = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColS = 128, kColP = 320;

}  // namespace

// Shared-memory layout, in bytes from a 1024-byte aligned base.
struct UmmaLayout {
  uint32_t q, info, bars, tmem_slot, total;
};

__host__ __device__ inline UmmaLayout umma_layout(int NS) {
  UmmaLayout L;
  L.q = static_cast<uint32_t>(NS) * 2u * kUTileBytes;  // stages first
  L.info = L.q + static_cast<uint32_t>(kUQBufs) * kUQBytes;  // the query buffers
  L.bars = L.info + static_cast<uint32_t>(NS) * sizeof(TileInfo);
  L.bars = (L.bars + 7u) & ~7u;
  const uint32_t nbars = 3u * NS + 17u;
  L.tmem_slot = L.bars + nbars * 8u;
  L.total = L.tmem_slot + 16u;
  return L;
}

// A bounded wait whose outcome is the same on every lane of the warp, so a
// warp never splits around the warp-wide tensor-memory loads and stores.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int32_t* err) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, err));
}

template <bool kBF16>
__global__ void __launch_bounds__(kUThreads, 1)
    pa_decode_umma_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmQ, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int NS = p.stages;
  const UmmaLayout Lay = umma_layout(NS);
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + Lay.info);
  const uint32_t base = smem_u32(smem);
  const uint32_t bar0 = base + Lay.bars;
  auto full_k = [&](int s) { return bar0 + 8u * s; };
  auto full_v = [&](int s) { return bar0 + 8u * (NS + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * NS + s); };
  const uint32_t barx = bar0 + 8u * (3 * NS);
  auto q_full = [&](int b) { return barx + 8u * b; };
  auto q_free = [&](int b) { return barx + 8u * (2 + b); };
  auto s_full = [&](int j) { return barx + 8u * (4 + j); };
  auto s_free = [&](int j) { return barx + 8u * (7 + j); };
  auto p_full = [&](int j) { return barx + 8u * (10 + j); };
  auto pv_done = [&](int j) { return barx + 8u * (13 + j); };
  const uint32_t o_free = barx + 8u * 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay.tmem_slot);
  // stage s: K rows (d-chunk dc, head g, token t) at ((dc * 4 + g) * 16 + t) * 128,
  // V the same 16 KiB further on
  auto k_addr = [&](int s) { return base + static_cast<uint32_t>(s) * 2u * kUTileBytes; };
  auto v_addr = [&](int s) { return k_addr(s) + kUTileBytes; };
  // query buffer qb: rows (d-chunk dc, head h, column c) at ((dc * 4 + h) * 32 + c) * 128
  auto q_addr = [&](int qb) { return base + Lay.q + static_cast<uint32_t>(qb) * kUQBytes; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hg = blockIdx.y;
  const int c = p.cta_base + blockIdx.x;  // this CTA's share of the line (LineCut)

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full_k(s), 1);
      mbar_init(full_v(s), 1);
      mbar_init(empty(s), 1);      // the P.V issuer's commit after the tile's products
    }
    for (int b = 0; b < kUQBufs; ++b) {
      mbar_init(q_full(b), 1);
      mbar_init(q_free(b), 1);     // the S issuer's commit
    }
    for (int b = 0; b < kUBufs; ++b) {
      mbar_init(s_full(b), 1);     // the S issuer's commit
      mbar_init(s_free(b), kUH);   // the four softmax warps
      mbar_init(p_full(b), kUH);
      mbar_init(pv_done(b), 1);    // the P.V issuer's commit
    }
    mbar_init(o_free, kUH);
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmQ);
  }
  if (warp == 5) {  // the whole warp allocates; the address lands in shared memory
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp < kUH) {
    // P is block diagonal: a row's weights sit in its own head's 8 columns of
    // every P buffer, the other 24 columns stay zero from here on
    const uint32_t zero[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    const uint32_t lrow = tmem + (static_cast<uint32_t>(32 * warp) << 16);
#pragma unroll
    for (int k = 0; k < kUBufs * 4; ++k) tmem_st16(lrow + kColP + 16u * k, zero);
    tmem_wait_st();
  }
  griddep_wait();  // the plan (and all earlier work on the stream) is complete
  // the next launch may start now: what it reads before its own wait, the
  // plan, is complete
  griddep_launch_dependents();

  int64_t lo = 0, hi = 0;
  if (host_plan_matches(p)) {
    lo = p.cta_lo[c];
    hi = p.cta_lo[c + 1];
  } else if (threadIdx.x == 0 && c == 0 && hg == 0) {
    flag_error(p.err, PA_DEVERR_BAD_PLAN);
  }
  const int G = p.group;

  if (lo < hi) {
    if (warp == 4) {
      // ======================= producer =======================
      if (lane == 0) {
        int32_t last_n = -1;
        produce_tiles<kUH, 2>(
            p, &tmK, &tmV, base, kUTileBytes, info, full_k(0), full_v(0), empty(0), NS, lo, hi,
            c, hg, false, [&](int32_t n, int32_t qrow0) {
              const int qb = n % kUQBufs;
              if (n >= kUQBufs &&
                  !mbar_wait(q_free(qb), static_cast<uint32_t>((n - kUQBufs) / kUQBufs) & 1u,
                             p.err))
                return false;
              // one box per (head, d-chunk): 32 / G query rows of the G query
              // heads of KV head h, i.e. the entry's 32 columns of that head
              mbar_arrive_expect_tx(q_full(qb), kUQBytes);
              for (int h = 0; h < kUH; ++h)
                for (int dc = 0; dc < 2; ++dc)
                  tma_load_4d(q_addr(qb) + (static_cast<uint32_t>(dc * kUH + h) * 32u) * 128u,
                              &tmQ, q_full(qb), 0, dc, (hg * kUH + h) * G, qrow0);
              last_n = n;
              return true;
            });
        // the last query loads (one per buffer) have landed before the CTA retires
        for (int32_t n = last_n >= kUQBufs ? last_n - kUQBufs + 1 : 0; n <= last_n; ++n)
          if (!mbar_wait(q_full(n % kUQBufs), static_cast<uint32_t>(n / kUQBufs) & 1u, p.err))
            break;
      }
    } else if (warp == 5) {
      // ======================= S issuer =======================
      if (lane == 0) {
        const uint32_t idS = idesc_f16(kBF16, 128, 64, false, false);
        int32_t n_entry = -1;
        for (int64_t t = lo; t < hi; ++t) {
          const int64_t u = t - lo;
          const int s = static_cast<int>(u % NS), j = static_cast<int>(u % kUBufs);
          if (!mbar_wait(full_k(s), static_cast<uint32_t>((u / NS) & 1), p.err)) break;
          if (info[s].flags & kNewSeq) {
            ++n_entry;
            // the previous entry's query buffer is free once its products finish
            if (n_entry >= 1) umma_commit(q_free((n_entry - 1) % kUQBufs));
            if (!mbar_wait(q_full(n_entry % kUQBufs), static_cast<uint32_t>(n_entry / kUQBufs) & 1u,
                           p.err))
              break;
          }
          if (u >= kUBufs &&
              !mbar_wait(s_free(j), static_cast<uint32_t>((u / kUBufs - 1) & 1), p.err))
            break;
          tc_fence_after();
          const uint32_t qa = q_addr(n_entry % kUQBufs), ka = k_addr(s);
          const uint32_t d = tmem + kColS + static_cast<uint32_t>(j) * 64u;
#pragma unroll
          for (int kc = 0; kc < 8; ++kc) {
            // d-chunk kc / 4 (the 128 rows of Q, the 64 rows of K, 1024-byte
            // 8-row groups), 16 elements at (kc % 4) * 32 bytes of each row
            const uint32_t dc = static_cast<uint32_t>(kc >> 2);
            const uint64_t a = smem_desc(qa + dc * 16384u + (kc & 3) * 32u, 16u, 1024u, kSwizzle128);
            const uint64_t b = smem_desc(ka + dc * 8192u + (kc & 3) * 32u, 16u, 1024u, kSwizzle128);
            umma_f16_ss(d, a, b, idS, kc > 0);
          }
          umma_commit(s_full(j));
        }
      }
    } else if (warp == 6) {
      // ======================= P.V issuer =======================
      if (lane == 0) {
        const uint32_t idPV = idesc_f16(kBF16, 128, 128, false, true);
        uint32_t ofree_par = 0;
        bool first_seg = true;
        int64_t pv_issued = -1;  // local index of the last P.V issued
        for (int64_t t = lo; t < hi; ++t) {
          const int64_t u = t - lo;
          const int s = static_cast<int>(u % NS), j = static_cast<int>(u % kUBufs);
          if (!mbar_wait(p_full(j), static_cast<uint32_t>((u / kUBufs) & 1), p.err)) break;
          const bool seg_start = (info[s].flags & kSegStart) != 0;
          if (seg_start) {
            // the previous segment's epilogue has read the accumulator
            if (!first_seg) {
              if (!mbar_wait(o_free, ofree_par, p.err)) break;
              ofree_par ^= 1u;
            }
            first_seg = false;
          }
          if (!mbar_wait(full_v(s), static_cast<uint32_t>((u / NS) & 1), p.err)) break;
          tc_fence_after();
#pragma unroll
          for (int part = 0; part < 2; ++part) {
#pragma unroll
            for (int g = 0; g < kUH; ++g) {
              // K step g: the 16 tokens of head g.  A: P columns of head g (8
              // tensor-memory columns); B: V[16 tokens x 128] of head g,
              // head_dim contiguous (MN-major), its d-chunks 8 KiB apart and
              // its 8-token row groups 1024 bytes apart
              const uint32_t a = tmem + kColP + static_cast<uint32_t>(j * 2 + part) * 32u +
                                 static_cast<uint32_t>(g) * 8u;
              const uint64_t b =
                  smem_desc(v_addr(s) + static_cast<uint32_t>(g) * 2048u, 8192u, 1024u,
                            kSwizzle128);
              umma_f16_ts(tmem + kColO, a, b, idPV, !(seg_start && part == 0 && g == 0));
            }
          }
          umma_commit(empty(s));
          umma_commit(pv_done(j));
          pv_issued = u;
        }
        // the last products have finished before tensor memory is released
        if (pv_issued >= 0)
          mbar_wait(pv_done(static_cast<int>(pv_issued % kUBufs)),
                    static_cast<uint32_t>((pv_issued / kUBufs) & 1), p.err);
      }
    } else if (warp == 7) {
      // ======================= pack tables =======================
      check_pack_tables(p, lo, hi, c, lane, 32);
    } else if (warp < kUH) {
      // ======================= softmax + epilogue =======================
      const int h = warp;        // KV head inside the CTA (= tensor-memory sub-partition)
      const int col = lane;      // query column = the row (h, col) of every product
      const int kvh = hg * kUH + h;
      const uint32_t lrow = tmem + (static_cast<uint32_t>(32 * h) << 16);
      const uint32_t tS = lrow + kColS + static_cast<uint32_t>(h) * 16u;  // + j * 64
      const uint32_t tP = lrow + kColP + static_cast<uint32_t>(h) * 8u;   // + (j * 2 + part) * 32
      const uint32_t tO = lrow + kColO;
      const float sl2 = p.scale_log2;
      const int cdiv = col / G;  // query row of this column inside the entry
      float m_run = -INFINITY, l_run = 0.f;
      for (int64_t t = lo; t < hi; ++t) {
        const int64_t u = t - lo;
        const int s = static_cast<int>(u % NS), j = static_cast<int>(u % kUBufs);
        const uint32_t ph = static_cast<uint32_t>((u / NS) & 1);
        const uint32_t bph = static_cast<uint32_t>((u / kUBufs) & 1);  // this buffer's use
        if (!warp_wait(full_k(s), ph, p.err)) break;
        const TileInfo ti = info[s];
        if (!warp_wait(s_full(j), bph, p.err)) break;
        tc_fence_after();
        uint32_t sr[16];
        tmem_ld16(tS + static_cast<uint32_t>(j) * 64u, sr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free(j));

        if (ti.flags & kSegStart) {
          m_run = -INFINITY;
          l_run = 0.f;
        }
        const uint32_t msk = static_cast<uint32_t>(ti.mask);
        // Every token of the tile visible to every column (the common case):
        // no per-token selection.  Columns past the entry's (other queries or
        // zero rows) are computed like the others and never written.
        const bool full = __all_sync(
            0xffffffffu, msk == 0xffffu && (!(ti.flags & kCausal) || ti.rel + cdiv >= kTile - 1));
        float x[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) x[k] = __uint_as_float(sr[k]);
        float mx;
        if (full) {
          float m8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = fmaxf(x[k], x[k + 8]);
#pragma unroll
          for (int k = 0; k < 4; ++k) m8[k] = fmaxf(m8[k], m8[k + 4]);
          mx = fmaxf(fmaxf(m8[0], m8[2]), fmaxf(m8[1], m8[3])) * sl2;
        } else {
          // column c sees tile rows up to rel + c / G (rel = 16: all)
          const int lim = (ti.flags & kCausal) ? ti.rel + cdiv : kTile;
          mx = -INFINITY;
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const bool ok = ((msk >> k) & 1u) && k <= lim;
            x[k] = ok ? x[k] * sl2 : -INFINITY;
            mx = fmaxf(mx, x[k]);
          }
        }
        // the running maximum moves only when exceeded by 2^kLazyLog2
        bool rescale = false;
        float alpha = 1.f;
        if (mx > m_run + kLazyLog2) {
          if (m_run != -INFINITY) {
            rescale = true;
            alpha = ex2(m_run - mx);
          }
          m_run = mx;
        }
        if (__any_sync(0xffffffffu, rescale)) {
          // this row's accumulator holds earlier tiles of the segment: wait for
          // the last products into it (tile u - 1), then scale it in place
          if (!warp_wait(pv_done(static_cast<int>((u - 1) % kUBufs)),
                         static_cast<uint32_t>(((u - 1) / kUBufs) & 1), p.err))
            break;
          tc_fence_after();
#pragma unroll 1
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t o[16];
            tmem_ld16(tO + static_cast<uint32_t>(kk) * 16u, o);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(tO + static_cast<uint32_t>(kk) * 16u, o);
          }
          tmem_wait_st();
        }
        float pw[16];
        if (full) {
          const float nm = -m_run;
#pragma unroll
          for (int k = 0; k < 16; ++k) pw[k] = ex2(fmaf(x[k], sl2, nm));
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) pw[k] = x[k] == -INFINITY ? 0.f : ex2(x[k] - m_run);
        }
        float ps[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) ps[k] = pw[k] + pw[k + 8];
#pragma unroll
        for (int k = 0; k < 4; ++k) ps[k] += ps[k + 4];
        const float psum = (ps[0] + ps[2]) + (ps[1] + ps[3]);
        uint32_t phi[8], plo[8];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const float p0 = pw[k], p1 = pw[k + 1];
          if constexpr (kBF16) {
            // hi: the upper 16 bits of each fp32 weight (a bf16 value, by
            // truncation); lo: the exact remainder rounded to bf16
            const uint32_t u0 = __float_as_uint(p0) & 0xffff0000u;
            const uint32_t u1 = __float_as_uint(p1) & 0xffff0000u;
            phi[k >> 1] = (u0 >> 16) | u1;
            plo[k >> 1] = pack2<true>(p0 - __uint_as_float(u0), p1 - __uint_as_float(u1));
          } else {
            const uint32_t hh = pack2<false>(p0, p1);
            phi[k >> 1] = hh;
            plo[k >> 1] =
                pack2<false>(p0 - lo_to_float<false>(hh), p1 - hi_to_float<false>(hh));
          }
        }
        l_run = l_run * alpha + psum;
        // P buffer j was last read by the products of tile u - kUBufs
        if (u >= kUBufs && !warp_wait(pv_done(j), bph ^ 1u, p.err)) break;
        tmem_st8(tP + static_cast<uint32_t>(j * 2) * 32u, phi);
        tmem_st8(tP + static_cast<uint32_t>(j * 2 + 1) * 32u, plo);
        tmem_wait_st();
        if (msk != 0xffffu) {
          // tokens left out of the tile (past the sequence, or of a bad block)
          // may hold anything, NaN included, and every row's product reads
          // every head's V: zero those V rows, never multiply
          if (!warp_wait(full_v(s), ph, p.err)) break;
          const int i = h * 32 + lane;  // one (d-chunk, head, token) row each
          const int dc = i >> 6, g2 = (i >> 4) & 3, tok = i & 15;
          if (!((msk >> tok) & 1u)) {
            const uint32_t a = v_addr(s) + static_cast<uint32_t>((dc * kUH + g2) * 16 + tok) * 128u;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a + q * 16u), "r"(0u)
                           : "memory");
          }
          fence_async_smem();  // the zeroed rows are read by the tensor cores
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(j));

        if (ti.flags & kSegEnd) {
          if (!warp_wait(pv_done(j), bph, p.err)) break;
          tc_fence_after();
          const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
          const bool direct = (ti.flags & kDirect) != 0;
          const bool part_ok = direct || ti.seg < p.nseg_cap;
          if (!direct && !part_ok && lane == 0) flag_error(p.err, PA_DEVERR_BAD_SEQLEN);
          const bool col_ok = col < ti.members * G;
          const int r = cdiv;
          const int64_t orow =
              (static_cast<int64_t>(ti.qrow0) + r) * p.num_q_heads + kvh * G + (col - r * G);
          const int64_t prow = part_row(p, ti.seg, kvh, col);
#pragma unroll 1
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t o[16];
            tmem_ld16(tO + static_cast<uint32_t>(kk) * 16u, o);
            if (!col_ok || !part_ok) continue;
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(o[i]) * inv;
            if (direct && !p.out_vec16) {  // an output view off 16-byte alignment
              for (int i = 0; i < 16; ++i) {
                const int64_t o2 = orow * kUD + kk * 16 + i;
                if (p.out_dtype == PA_F32)
                  static_cast<float*>(p.out)[o2] = v[i];
                else if (p.out_dtype == PA_BF16)
                  static_cast<__nv_bfloat16*>(p.out)[o2] = __float2bfloat16_rn(v[i]);
                else
                  static_cast<__half*>(p.out)[o2] = __float2half_rn(v[i]);
              }
            } else if (direct) {
              if (p.out_dtype == PA_F32) {
                float4* op = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * kUD +
                                                       kk * 16);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  op[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
              } else {
                uint32_t w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                  w[i] = p.out_dtype == PA_BF16 ? pack2<true>(v[2 * i], v[2 * i + 1])
                                                : pack2<false>(v[2 * i], v[2 * i + 1]);
                uint4* op = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow * kUD +
                                                     kk * 16);
                op[0] = make_uint4(w[0], w[1], w[2], w[3]);
                op[1] = make_uint4(w[4], w[5], w[6], w[7]);
              }
            } else {
              float4* op = reinterpret_cast<float4*>(p.part_o + prow * kUD + kk * 16);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                op[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
          }
          if (!direct && part_ok && col_ok) {
            p.part_ml[prow * 2] = l_run > 0.f ? m_run : -INFINITY;
            p.part_ml[prow * 2 + 1] = l_run;
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free);
        }
      }
    }
  }
  // teardown: every warp is here once its last wait has ended (each is
  // bounded), so the products have finished and tensor memory can go back
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
UmmaKernel select_umma(bool bf16) {
  return bf16 ? pa_decode_umma_kernel<true> : pa_decode_umma_kernel<false>;
}

size_t umma_smem_bytes(int stages) { return 1024u + umma_layout(stages).total; }

}  // namespace pa
