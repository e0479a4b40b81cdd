// pa_decode_umma.cu -- the decode main kernel on the fifth-generation tensor
// cores (tcgen05, tensor memory), for entries with many query columns: packs
// of samples over a shared prompt ("PagedAttention", "Sharing and
// copy-on-write": the samples' tables point at the same prompt blocks, so a
// block read once serves every sample's query) and chunks of several query
// tokens of one sequence.  Same plan, tile line, segments, partials and
// combine as the warp-level kernel of pa_decode.cu; only the consumer side
// differs.
//
// Per KV head g of the CTA's HG heads and per 16-token tile of an entry:
//   S[c, t]  = Q[c, :] . K[t, :]   one 64 x 16 x 128 product (eight K=16
//                                   MMAs), the entry's up to 32 query
//                                   columns c on M (rows 32..63 are never
//                                   read), the tile's tokens on N, into
//                                   tensor memory;
//   online softmax of each row c by the thread owning that accumulator row:
//                                   no cross-thread reduction; the running
//                                   maximum moves only when a tile's maximum
//                                   exceeds it by 2^8, so the accumulator is
//                                   rarely rescaled; P = hi + lo (two 16-bit
//                                   halves) written to shared memory;
//   O[c, :] += P[c, :] . V[:, :]   two 64 x 128 x 16 products (hi and lo)
//                                   accumulating in tensor memory.
// The 64-row accumulators take half of each tensor-memory sub-partition, so
// the KV heads of the CTA pair up: head 2r in lanes 0..15 and head 2r + 1 in
// lanes 16..31 of sub-partitions 0 and 1, region r of the columns.
//
// Warps: 0, 1, 4, 5 softmax and epilogue (sub-partitions 0 and 1 of regions
// 0 and 1), 2 producer (TMA: K/V tiles and each entry's query rows), 3 and 6
// issue the S products of regions 0 and 1, 7 issues every P.V product.  One
// thread issues a tcgen05.mma about every 60 cycles, while several issuing
// warps overlap (measured on B200), so the small S products are spread over
// two issuers and run ahead of the softmax (two S buffers per region), and the
// P.V products follow it on their own.  Warp 3 owns the tensor memory.  Every
// wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>

#include "pa_decode_common.cuh"
#include "pa_device.cuh"
#include "pa_umma.cuh"

namespace pa {

namespace {

constexpr int kUD = 128;             // head_dim of this kernel
constexpr int kUThreads = kUmmaThreads;  // 8 warps
constexpr float kLazyLog2 = 8.0f;    // growth of a row maximum that forces a rescale
constexpr uint32_t kQBlock = 32 * 128;   // 32 query rows of one (head, d-chunk): 4 KiB
constexpr uint32_t kPBlock = 32 * 32;    // 32 rows of 16 tokens of P, one half: 1 KiB

}  // namespace

// Shared-memory layout, in bytes from a 1024-byte aligned base.
struct UmmaLayout {
  uint32_t stage, q, p, info, bars, tmem_slot, total;
};

__host__ __device__ inline UmmaLayout umma_layout(int HG, int NS) {
  UmmaLayout L;
  const uint32_t tile = static_cast<uint32_t>(kTile * HG * kUD * 2);
  L.stage = 0;
  L.q = static_cast<uint32_t>(NS) * 2u * tile;
  // two query buffers; the M = 64 operands read 32 rows past the last block
  L.p = L.q + 2u * HG * 2u * kQBlock + kQBlock;
  // two P buffers x HG heads x (hi, lo); again 32 rows past the last block
  L.info = L.p + 2u * HG * 2u * kPBlock + kPBlock;
  L.bars = L.info + static_cast<uint32_t>(NS) * sizeof(TileInfo);
  L.bars = (L.bars + 7u) & ~7u;
  const uint32_t nbars = 3u * NS + 19u;
  L.tmem_slot = L.bars + nbars * 8u;
  L.total = L.tmem_slot + 16u;
  return L;
}

// A bounded wait whose outcome is the same on every lane of the warp, so a
// warp never splits around the warp-wide tensor-memory loads and stores.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, int32_t* err) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, err));
}

template <int HG, bool kBF16>
__global__ void __launch_bounds__(kUThreads, 1)
    pa_decode_umma_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmQ, const DecodeParams p) {
  static_assert(HG == 2 || HG == 4, "two or four KV heads per CTA");
  constexpr int R = HG / 2;                 // tensor-memory regions (two heads each)
  constexpr uint32_t kTileBytes = kTile * HG * kUD * 2;
  constexpr uint32_t kTmemCols = HG == 4 ? 512u : 256u;
  constexpr uint32_t kSCol0 = R * 128u;     // S buffers after the O accumulators

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int NS = p.stages;
  const UmmaLayout Lay = umma_layout(HG, NS);
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + Lay.info);
  const uint32_t base = smem_u32(smem);
  const uint32_t bar0 = base + Lay.bars;
  auto full_k = [&](int s) { return bar0 + 8u * s; };
  auto full_v = [&](int s) { return bar0 + 8u * (NS + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * NS + s); };
  const uint32_t barx = bar0 + 8u * (3 * NS);
  auto q_full = [&](int b) { return barx + 8u * b; };
  auto q_free = [&](int b) { return barx + 8u * (2 + b); };
  auto p_full = [&](int j) { return barx + 8u * (4 + j); };
  auto pv_done = [&](int j) { return barx + 8u * (6 + j); };
  const uint32_t o_free = barx + 8u * 8;
  auto s_full = [&](int r, int j) { return barx + 8u * (9 + 2 * r + j); };
  auto s_free = [&](int r, int j) { return barx + 8u * (13 + 2 * r + j); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay.tmem_slot);
  auto q_addr = [&](int qb, int g, int dc) {
    return base + Lay.q + ((static_cast<uint32_t>(qb) * HG + g) * 2u + dc) * kQBlock;
  };
  auto p_addr = [&](int j, int g, int part) {
    return base + Lay.p + ((static_cast<uint32_t>(j) * HG + g) * 2u + part) * kPBlock;
  };
  auto k_addr = [&](int s) { return base + static_cast<uint32_t>(s) * 2u * kTileBytes; };
  auto v_addr = [&](int s) { return k_addr(s) + kTileBytes; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hg = blockIdx.y;
  const int c = blockIdx.x;
  const int64_t C = p.ctas_per_group;
  constexpr int NSW = 2 * R;  // softmax warps
  const bool is_softmax = (warp & 3) < 2 && (warp >> 2) < R;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(full_k(s), 1);
      mbar_init(full_v(s), 1);
      mbar_init(empty(s), 1);  // the P.V issuer's commit after the tile's products
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(q_full(b), 1);
      mbar_init(q_free(b), R);        // each S issuer's commit
      mbar_init(p_full(b), NSW);      // every softmax warp's P rows
      mbar_init(pv_done(b), 1);       // the P.V issuer's commit
      for (int r = 0; r < 2; ++r) {
        mbar_init(s_full(r, b), 1);   // S issuer r's commit
        mbar_init(s_free(r, b), 2);   // region r's two softmax warps
      }
    }
    mbar_init(o_free, NSW);
    fence_mbar_init();
  }
  if (warp == 2 && lane == 0) {
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmQ);
  }
  if (warp == 3) {  // the whole warp allocates; the address lands in shared memory
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();
  griddep_wait();  // the plan (and all earlier work on the stream) is complete

  int64_t lo = 0, hi = 0;
  if (host_plan_matches(p)) {
    const int E = p.meta[1];
    const int64_t N = p.plan_tiles[E];
    lo = static_cast<int64_t>(c) * N / C;
    hi = static_cast<int64_t>(c + 1) * N / C;
  } else if (threadIdx.x == 0 && c == 0 && hg == 0) {
    flag_error(p.err, PA_DEVERR_BAD_PLAN);
  }
  const int TB = p.tok_box;
  // K operand (N = 16 tokens): 8-token row groups 1024 bytes apart in a
  // 16-token box, or one box of HG x 2 x 8 rows apart with 8-token boxes
  const uint32_t sbo_tok = TB == 16 ? 1024u : static_cast<uint32_t>(HG) * 2048u;
  const int G = p.group;

  if (lo < hi) {
    if (warp == 2) {
      // ======================= producer =======================
      if (lane == 0) {
        int32_t last_n = -1;
        produce_tiles<HG, 2>(
            p, &tmK, &tmV, base, kTileBytes, info, full_k(0), full_v(0), empty(0), NS, lo, hi,
            c, hg, false, [&](int32_t n, int32_t qrow0) {
              const int qb = n & 1;
              if (n >= 2 && !mbar_wait(q_free(qb), static_cast<uint32_t>((n - 2) >> 1) & 1u, p.err))
                return false;
              mbar_arrive_expect_tx(q_full(qb), HG * 2u * kQBlock);
              for (int g = 0; g < HG; ++g)
                for (int dc = 0; dc < 2; ++dc)
                  tma_load_4d(q_addr(qb, g, dc), &tmQ, q_full(qb), 0, dc, (hg * HG + g) * G,
                              qrow0);
              last_n = n;
              return true;
            });
        // the last (up to two) query loads have landed before the CTA retires
        for (int32_t n = last_n > 0 ? last_n - 1 : 0; n <= last_n; ++n)
          if (!mbar_wait(q_full(n & 1), static_cast<uint32_t>(n >> 1) & 1u, p.err)) break;
      }
    } else if ((warp == 3 || warp == 6) && (warp == 3 || R == 2)) {
      // ======================= S issuer of region r =======================
      if (lane == 0) {
        const int r = warp == 3 ? 0 : 1;
        const uint32_t idS = idesc_f16(kBF16, 64, 16, false, false);
        int32_t n_entry = -1;
        for (int64_t t = lo; t < hi; ++t) {
          const int64_t u = t - lo;
          const int s = static_cast<int>(u % NS), j = static_cast<int>(u & 1);
          if (!mbar_wait(full_k(s), static_cast<uint32_t>((u / NS) & 1), p.err)) break;
          if (info[s].flags & kNewSeq) {
            ++n_entry;
            // the previous entry's query buffer is free once its products finish
            if (n_entry >= 1) umma_commit(q_free((n_entry - 1) & 1));
            if (!mbar_wait(q_full(n_entry & 1), static_cast<uint32_t>(n_entry >> 1) & 1u, p.err))
              break;
          }
          if (u >= 2 &&
              !mbar_wait(s_free(r, j), static_cast<uint32_t>((u - 2) >> 1) & 1u, p.err))
            break;
          tc_fence_after();
          const int qb = n_entry & 1;
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const int g = 2 * r + gg;
            const uint32_t d = tmem + (static_cast<uint32_t>(gg * 16) << 16) + kSCol0 +
                               static_cast<uint32_t>(r) * 32u + static_cast<uint32_t>(j) * 16u;
#pragma unroll
            for (int kc = 0; kc < 8; ++kc) {
              const uint64_t a =
                  smem_desc(q_addr(qb, g, kc >> 2) + (kc & 3) * 32u, 16u, 1024u, kSwizzle128);
              const uint64_t b = smem_desc(
                  k_addr(s) + static_cast<uint32_t>((g * 2 + (kc >> 2)) * TB) * 128u +
                      (kc & 3) * 32u,
                  16u, sbo_tok, kSwizzle128);
              umma_f16_ss(d, a, b, idS, kc > 0);
            }
          }
          umma_commit(s_full(r, j));
        }
      }
    } else if (warp == 7) {
      // ======================= P.V issuer =======================
      if (lane == 0) {
        const uint32_t idPV = idesc_f16(kBF16, 64, 128, false, true);
        uint32_t ofree_par = 0;
        bool first_seg = true;
        int64_t pv_issued = -1;  // local index of the last P.V issued
        for (int64_t t = lo; t < hi; ++t) {
          const int64_t u = t - lo;
          const int s = static_cast<int>(u % NS), j = static_cast<int>(u & 1);
          if (!mbar_wait(p_full(j), static_cast<uint32_t>(u >> 1) & 1u, p.err)) break;
          const bool seg_start = (info[s].flags & kSegStart) != 0;
          if (seg_start) {
            // the previous segment's epilogue has read its accumulator
            if (!first_seg) {
              if (!mbar_wait(o_free, ofree_par, p.err)) break;
              ofree_par ^= 1u;
            }
            first_seg = false;
          }
          if (!mbar_wait(full_v(s), static_cast<uint32_t>((u / NS) & 1), p.err)) break;
          tc_fence_after();
#pragma unroll
          for (int g = 0; g < HG; ++g) {
            const uint32_t d = tmem + (static_cast<uint32_t>((g & 1) * 16) << 16) +
                               static_cast<uint32_t>(g >> 1) * 128u;
            // V[16 tokens x 128]: N = head_dim contiguous (MN-major), d-chunks
            // TB rows apart, 8-token row groups sbo_tok apart
            const uint64_t b =
                smem_desc(v_addr(s) + static_cast<uint32_t>(g * 2 * TB) * 128u,
                          static_cast<uint32_t>(TB) * 128u, sbo_tok, kSwizzle128);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
              // P[64 x 16], K-major without swizzle: 8-row core matrices of
              // 16 bytes, tokens 8..15 128 bytes on, row groups 256 apart
              const uint64_t a = smem_desc(p_addr(j, g, part), 128u, 256u, kSwizzleNone);
              umma_f16_ss(d, a, b, idPV, !(seg_start && part == 0));
            }
          }
          umma_commit(empty(s));
          umma_commit(pv_done(j));
          pv_issued = u;
        }
        // the last products have finished before tensor memory is released
        if (pv_issued >= 0)
          mbar_wait(pv_done(static_cast<int>(pv_issued & 1)),
                    static_cast<uint32_t>(pv_issued >> 1) & 1u, p.err);
      }
    } else if (is_softmax) {
      // ======================= softmax + epilogue =======================
      const int region = warp >> 2, sub = warp & 3;
      const int sw = region * 2 + sub;              // softmax warp 0 .. NSW - 1
      const int g = 2 * region + (lane >> 4);       // KV head inside the CTA
      const int col = sub * 16 + (lane & 15);       // query column = accumulator row
      const int kvh = hg * HG + g;
      const uint32_t lane_field = static_cast<uint32_t>(32 * sub) << 16;
      const uint32_t tS = tmem + lane_field + kSCol0 + static_cast<uint32_t>(region) * 32u;
      const uint32_t tO = tmem + lane_field + static_cast<uint32_t>(region) * 128u;
      const float sl2 = p.scale_log2;
      float m_run = -INFINITY, l_run = 0.f;
      for (int64_t t = lo; t < hi; ++t) {
        const int64_t u = t - lo;
        const int s = static_cast<int>(u % NS), j = static_cast<int>(u & 1);
        const uint32_t ph = static_cast<uint32_t>((u / NS) & 1);
        if (!warp_wait(full_k(s), ph, p.err)) break;
        const TileInfo ti = info[s];
        if (!warp_wait(s_full(region, j), static_cast<uint32_t>(u >> 1) & 1u, p.err)) break;
        tc_fence_after();
        uint32_t sr[16];
        tmem_ld16(tS + static_cast<uint32_t>(j) * 16u, sr);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free(region, j));

        if (ti.flags & kSegStart) {
          m_run = -INFINITY;
          l_run = 0.f;
        }
        const int ncol = ti.members * G;
        const bool col_ok = col < ncol;
        // column c sees tile rows up to rel + c / G (rel = 16: all)
        const int lim = (ti.flags & kCausal) ? ti.rel + col / G : kTile;
        const uint32_t msk = static_cast<uint32_t>(ti.mask);
        float sv[16];
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const bool ok = col_ok && ((msk >> k) & 1u) && k <= lim;
          sv[k] = ok ? __uint_as_float(sr[k]) * sl2 : -INFINITY;
          mx = fmaxf(mx, sv[k]);
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
          // the last product into it (tile u - 1), then scale it in place
          if (!warp_wait(pv_done(static_cast<int>((u - 1) & 1)),
                         static_cast<uint32_t>((u - 1) >> 1) & 1u, p.err))
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
        float psum = 0.f;
        uint32_t phi[8], plo[8];
#pragma unroll
        for (int k = 0; k < 16; k += 2) {
          const float p0 = sv[k] == -INFINITY ? 0.f : ex2(sv[k] - m_run);
          const float p1 = sv[k + 1] == -INFINITY ? 0.f : ex2(sv[k + 1] - m_run);
          psum += p0 + p1;
          const uint32_t h = pack2<kBF16>(p0, p1);
          phi[k >> 1] = h;
          plo[k >> 1] = pack2<kBF16>(p0 - lo_to_float<kBF16>(h), p1 - hi_to_float<kBF16>(h));
        }
        l_run = l_run * alpha + psum;
        // P buffer j was last read by the product of tile u - 2
        if (u >= 2 && !warp_wait(pv_done(j), static_cast<uint32_t>((u - 2) >> 1) & 1u, p.err))
          break;
        {
          const uint32_t r0 = static_cast<uint32_t>(col >> 3) * 256u + (col & 7) * 16u;
          const uint32_t ah = p_addr(j, g, 0) + r0, al = p_addr(j, g, 1) + r0;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ah), "r"(phi[0]),
                       "r"(phi[1]), "r"(phi[2]), "r"(phi[3]) : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(ah + 128u), "r"(phi[4]),
                       "r"(phi[5]), "r"(phi[6]), "r"(phi[7]) : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(al), "r"(plo[0]),
                       "r"(plo[1]), "r"(plo[2]), "r"(plo[3]) : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(al + 128u), "r"(plo[4]),
                       "r"(plo[5]), "r"(plo[6]), "r"(plo[7]) : "memory");
        }
        if (msk != 0xffffu) {
          // tokens left out of the tile (past the sequence, or of a bad block)
          // may hold anything, NaN included: zero their V rows, never multiply
          if (!warp_wait(full_v(s), ph, p.err)) break;
          const int i = sw * 32 + lane;  // one (head, d-chunk, token) row each
          const int g2 = i >> 5, dc = (i >> 4) & 1, tok = i & 15;
          if (g2 < HG && !((msk >> tok) & 1u)) {
            const uint32_t row =
                static_cast<uint32_t>(((tok / TB) * HG * 2 + g2 * 2 + dc) * TB + tok % TB);
            const uint32_t a = v_addr(s) + row * 128u;
#pragma unroll
            for (int q = 0; q < 8; ++q)
              asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a + q * 16u), "r"(0u)
                           : "memory");
          }
        }
        fence_async_smem();  // the P rows (and zeroed V rows) are read by the tensor cores
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full(j));

        if (ti.flags & kSegEnd) {
          if (!warp_wait(pv_done(j), static_cast<uint32_t>(u >> 1) & 1u, p.err)) break;
          tc_fence_after();
          const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
          const bool direct = (ti.flags & kDirect) != 0;
          const bool part_ok = direct || ti.seg < p.nseg_cap;
          if (!direct && !part_ok && lane == 0) flag_error(p.err, PA_DEVERR_BAD_SEQLEN);
          const int r = col / G;
          const int64_t orow =
              (static_cast<int64_t>(ti.qrow0) + r) * p.num_q_heads + kvh * G + (col - r * G);
          const int64_t prow =
              ((static_cast<int64_t>(hg) * p.nseg_cap + ti.seg) * HG + g) * p.cols + col;
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
                const int64_t o = orow * kUD + kk * 16 + i;
                if (p.out_dtype == PA_F32)
                  static_cast<float*>(p.out)[o] = v[i];
                else if (p.out_dtype == PA_BF16)
                  static_cast<__nv_bfloat16*>(p.out)[o] = __float2bfloat16_rn(v[i]);
                else
                  static_cast<__half*>(p.out)[o] = __float2half_rn(v[i]);
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
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
UmmaKernel select_umma(int HG, bool bf16) {
  if (HG == 4) return bf16 ? pa_decode_umma_kernel<4, true> : pa_decode_umma_kernel<4, false>;
  if (HG == 2) return bf16 ? pa_decode_umma_kernel<2, true> : pa_decode_umma_kernel<2, false>;
  return nullptr;
}

size_t umma_smem_bytes(int HG, int stages) {
  return 1024u + umma_layout(HG, stages).total;
}

}  // namespace pa
