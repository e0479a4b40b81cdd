// linecut_check.cu -- host-side check of how the decode cuts its tile line
// into CTA shares (LineCut in the decode kernels' common header), against
// the definition written out as loops.  Built by nvcc with the library's
// flags; runs on the CPU only (no kernel is launched).
//
// The definition: N tiles laid end to end, C CTA shares [lo(c), lo(c + 1)).
// One kernel (S = 0): lo(c) = floor(c N / C).  Split (0 < S < C): the first
// NK tiles (the packs' prefixes) are cut evenly over CTAs 0 .. S-1 and the
// other N - NK over CTAs S .. C-1.  count_below(x) is the number of CTAs
// whose share starts below tile x.
#include <cstdint>
#include <cstdio>
#include <cstdlib>

#include "../../paged_kv_cache_343_b200/csrc/pa_decode_common.cuh"

static int failures = 0;

static void expect(bool ok, const char* what, int64_t C, int64_t S, int64_t N, int64_t NK,
                   int64_t at) {
  if (!ok && failures < 20) {
    std::printf("FAIL %s: C=%lld S=%lld N=%lld NK=%lld at %lld\n", what, (long long)C,
                (long long)S, (long long)N, (long long)NK, (long long)at);
  }
  if (!ok) ++failures;
}

static void check(int64_t C, int64_t S, int64_t N, int64_t NK) {
  pa::LineCut cut;
  cut.C = C;
  cut.S = S;
  cut.N = N;
  cut.NK = NK;
  // the shares: contiguous, covering [0, N), even within each piece
  expect(cut.lo(0) == 0, "lo(0) == 0", C, S, N, NK, 0);
  expect(cut.lo(C) == N, "lo(C) == N", C, S, N, NK, C);
  int64_t min_a = INT64_MAX, max_a = -1, min_b = INT64_MAX, max_b = -1;
  for (int64_t c = 0; c < C; ++c) {
    const int64_t a = cut.lo(c), b = cut.lo(c + 1);
    expect(a <= b, "lo non-decreasing", C, S, N, NK, c);
    const int64_t len = b - a;
    if (S == 0 || c >= S) {
      if (len < min_b) min_b = len;
      if (len > max_b) max_b = len;
    } else {
      if (len < min_a) min_a = len;
      if (len > max_a) max_a = len;
    }
    // with a split no share mixes the packs' tiles and the sequences' tiles
    if (S > 0) expect(b <= NK || a >= NK, "share within one piece", C, S, N, NK, c);
  }
  if (S > 0) {
    expect(cut.lo(S) == NK, "lo(S) == NK", C, S, N, NK, S);
    expect(max_a - min_a <= 1, "even shares of the packs", C, S, N, NK, 0);
    expect(min_a * S <= NK && NK <= max_a * S, "pack shares sum to NK", C, S, N, NK, 0);
  }
  expect(max_b - min_b <= 1, "even shares", C, S, N, NK, 0);
  // count_below against a count over all CTAs
  for (int64_t x = 0; x <= N; ++x) {
    int64_t n = 0;
    for (int64_t c = 0; c < C; ++c) n += cut.lo(c) < x ? 1 : 0;
    expect(cut.count_below(x) == n, "count_below", C, S, N, NK, x);
  }
}

int main() {
  // the benchmark's shapes: llama8b (148 CTAs, 9652 tiles), the shared
  // prompt's split (74 + 148 CTAs, 4064 pack tiles, 2009 more)
  check(148, 0, 9652, 0);
  check(222, 74, 6073, 4064);
  // edges: no tiles, fewer tiles than CTAs, no packs, no sequence tiles
  check(148, 0, 0, 0);
  check(148, 0, 37, 0);
  check(222, 74, 2009, 0);
  check(222, 74, 4064, 4064);
  check(2, 1, 1, 1);
  check(3, 1, 5, 0);
  // random shapes
  uint64_t state = 12345;
  auto next = [&state](int64_t bound) {
    state = state * 6364136223846793005ull + 1442695040888963407ull;
    return static_cast<int64_t>((state >> 33) % static_cast<uint64_t>(bound));
  };
  for (int r = 0; r < 400; ++r) {
    const int64_t C = 1 + next(300);
    const int64_t S = (C > 1 && next(2)) ? 1 + next(C - 1) : 0;
    const int64_t N = next(3000);
    const int64_t NK = S > 0 ? next(N + 1) : 0;
    check(C, S, N, NK);
  }
  if (failures) {
    std::printf("%d checks failed\n", failures);
    return 1;
  }
  std::printf("all checks held\n");
  return 0;
}
