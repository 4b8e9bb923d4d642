// Host-side checks of the two stream-K planners of the exact-attention path
// (Eq. (3.1) of "Nectar: Neural Estimation of Cached-Token Attention via
// Regression", split over the n cached keys and joined by log-sum-exp), run
// on the CPU against the library's own objects: plan_decode and
// dec_smem_for_rows (attn_decode.cu), plan_tc (attn_tc.cu).
//
// Both kernels give CTA c of C the tiles [c T / C, (c + 1) T / C) of a list
// of T tiles.  From that definition alone this program counts, by brute
// force over the CTAs, what the planners claim:
//   split kernel   every CTA has at least one tile, and S_max (the partial
//                  slots a head gets in the workspace) is the largest number
//                  of CTAs whose range touches one head;
//   tensor cores   dp_rounds whole rounds of C units plus sk_units units cut
//                  by key tiles make up all units; a stream-K rest cuts at
//                  most the 2 units of each CTA's range it has partial slots
//                  for (the first and the last), a lockstep rest puts every
//                  key tile of its units in exactly one of at most 2 items
//                  per CTA, within 10 % of the even cut; the workspace holds
//                  2 slots of 256 rows of (d + 2) floats per CTA;
//   shared memory  every split launch fits 227 KB per CTA, and the launches
//                  bounded to two CTAs per SM fit the SM's 228 KB twice.
// Prints "ok <cases>" and exits 0, or prints the first failure and exits 1.
#include <cstdint>
#include <cstdio>
#include <vector>

#include "kernels.h"

namespace nectar {
// The planners' objects reference the C ABI's error text; nothing here sets it.
void set_last_error(const char*) {}
}  // namespace nectar

namespace {

constexpr int64_t kD = 128;
constexpr size_t kMaxSmemPerCta = 227 * 1024;
constexpr size_t kSmemPerSm = 228 * 1024;
constexpr size_t kReservedPerCta = 1024;   // the driver's per-CTA shared-memory reserve

int64_t g_cases = 0;

#define CHECK(cond, ...)                                  \
  do {                                                    \
    if (!(cond)) {                                        \
      std::printf("FAIL %s:%d: %s | ", __FILE__, __LINE__, #cond); \
      std::printf(__VA_ARGS__);                           \
      std::printf("\n");                                  \
      return false;                                       \
    }                                                     \
  } while (0)

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool check_decode(int heads, int64_t n, int sms, int cps, int tile) {
  ++g_cases;
  const nectar::DecPlan pl = nectar::plan_decode(heads, n, sms, cps, tile);
  CHECK(pl.tile == tile, "tile %d", pl.tile);
  CHECK(pl.tph == cdiv(n, tile), "heads %d n %lld tph %lld", heads, (long long)n, (long long)pl.tph);
  CHECK(pl.total == heads * pl.tph, "total %lld", (long long)pl.total);
  if (pl.total == 0) {
    CHECK(pl.S_max == 0 && pl.C >= 1, "empty plan C %d S_max %d", pl.C, pl.S_max);
    return true;
  }
  const int64_t want_c = std::min<int64_t>(static_cast<int64_t>(sms) * cps, pl.total);
  CHECK(pl.C == want_c, "heads %d n %lld sms %d cps %d: C %d want %lld", heads, (long long)n, sms, cps, pl.C,
        (long long)want_c);
  std::vector<int> touching(heads, 0);
  for (int64_t c = 0; c < pl.C; ++c) {
    const int64_t t0 = c * pl.total / pl.C, t1 = (c + 1) * pl.total / pl.C;
    CHECK(t1 > t0, "CTA %lld has no tile (T %lld C %d)", (long long)c, (long long)pl.total, pl.C);
    for (int64_t h = t0 / pl.tph; h <= (t1 - 1) / pl.tph; ++h) ++touching[h];
  }
  int most = 0;
  for (int h = 0; h < heads; ++h) most = std::max(most, touching[h]);
  CHECK(pl.S_max == most, "heads %d n %lld C %d: S_max %d, brute force %d", heads, (long long)n, pl.C, pl.S_max,
        most);
  return true;
}

bool check_tc(int heads, int64_t n, int64_t rows, int sms) {
  ++g_cases;
  constexpr int64_t kUnitRows = 256, kKeys = 64;
  const nectar::TcPlan pl = nectar::plan_tc(heads, n, rows, sms);
  CHECK(pl.qpairs == cdiv(rows, kUnitRows), "rows %lld qpairs %d", (long long)rows, pl.qpairs);
  CHECK(pl.tph == cdiv(n, kKeys), "n %lld tph %lld", (long long)n, (long long)pl.tph);
  const int64_t units = static_cast<int64_t>(heads) * pl.qpairs;
  CHECK(pl.C >= 1 && pl.C <= sms && pl.C <= std::max<int64_t>(1, units * pl.tph), "C %d", pl.C);
  CHECK(pl.dp_rounds >= 0 && pl.sk_units >= 0, "dp %d sk %lld", pl.dp_rounds, (long long)pl.sk_units);
  CHECK(static_cast<int64_t>(pl.dp_rounds) * pl.C + pl.sk_units == units, "dp %d x C %d + sk %lld != units %lld",
        pl.dp_rounds, pl.C, (long long)pl.sk_units, (long long)units);
  CHECK(pl.ws_bytes >= static_cast<size_t>(pl.C) * 2 * kUnitRows * (kD + 2) * sizeof(float), "ws %zu",
        pl.ws_bytes);
  CHECK(pl.smem <= kMaxSmemPerCta, "smem %zu", pl.smem);
  if (pl.sk_parts > 0) {
    // lockstep rest: every whole round, the rest (< C units) in S equal key
    // parts, item q * U + u on CTA item % C, slot item / C (two slots)
    const int64_t U = pl.sk_units, S = pl.sk_parts, items = U * S;
    CHECK(pl.qpairs > 1 && U > 0 && U < pl.C, "lockstep with qpairs %d, rest %lld, C %d", pl.qpairs, (long long)U,
          pl.C);
    CHECK(pl.dp_rounds == units / pl.C, "lockstep rounds %d, units %lld", pl.dp_rounds, (long long)units);
    CHECK(S <= pl.tph && items <= 2 * static_cast<int64_t>(pl.C), "S %lld items %lld C %d tph %lld", (long long)S,
          (long long)items, pl.C, (long long)pl.tph);
    // every key tile of every rest unit in exactly one (CTA, slot); no slot used twice
    std::vector<int> seen(static_cast<size_t>(U * pl.tph), 0);
    std::vector<int> slot_used(static_cast<size_t>(pl.C) * 2, 0);
    int64_t longest = 0;
    for (int64_t c = 0; c < pl.C; ++c) {
      int64_t tiles = 0;
      for (int j = 0; c + j * static_cast<int64_t>(pl.C) < items; ++j) {
        const int64_t item = c + j * static_cast<int64_t>(pl.C);
        const int64_t q = item / U, u = item % U;
        const int64_t k0 = q * pl.tph / S, k1 = (q + 1) * pl.tph / S;
        CHECK(k1 > k0, "empty part %lld of %lld (tph %lld)", (long long)q, (long long)S, (long long)pl.tph);
        CHECK(j < 2, "CTA %lld has a third item", (long long)c);
        ++slot_used[c * 2 + j];
        for (int64_t k = k0; k < k1; ++k) ++seen[u * pl.tph + k];
        tiles += k1 - k0;
      }
      longest = std::max(longest, tiles);
    }
    for (size_t i = 0; i < seen.size(); ++i)
      CHECK(seen[i] == 1, "rest tile %zu covered %d times", i, seen[i]);
    for (size_t i = 0; i < slot_used.size(); ++i) CHECK(slot_used[i] <= 1, "slot %zu used twice", i);
    // within 10 % of cutting the rest evenly over the CTAs
    const int64_t even = cdiv(U * pl.tph, pl.C);
    CHECK(longest * 10 <= even * 11, "longest CTA %lld tiles, even cut %lld", (long long)longest, (long long)even);
    return true;
  }
  // stream-K rest: whole rounds are taken only while at least one round of
  // units is left to cut, so no CTA idles through the stream-K part
  if (pl.sk_units > 0 && pl.dp_rounds > 0)
    CHECK(pl.sk_units >= pl.C && pl.sk_units < 2 * static_cast<int64_t>(pl.C), "sk %lld C %d",
          (long long)pl.sk_units, pl.C);
  const int64_t Tsk = pl.sk_units * pl.tph;
  for (int64_t c = 0; c < pl.C && Tsk > 0; ++c) {
    const int64_t s0 = c * Tsk / pl.C, s1 = (c + 1) * Tsk / pl.C;
    CHECK(s1 > s0, "CTA %lld has no key tile (Tsk %lld C %d)", (long long)c, (long long)Tsk, pl.C);
    int cut = 0;
    for (int64_t u = s0 / pl.tph; u <= (s1 - 1) / pl.tph; ++u) {
      const int64_t b = u * pl.tph, e = b + pl.tph;
      const bool whole = s0 <= b && s1 >= e;
      if (!whole) {
        ++cut;
        CHECK(u == s0 / pl.tph || u == (s1 - 1) / pl.tph, "CTA %lld cuts a middle unit %lld", (long long)c,
              (long long)u);
      }
    }
    CHECK(cut <= 2, "CTA %lld cuts %d units", (long long)c, cut);
  }
  return true;
}

bool check_smem() {
  for (int R = 1; R <= nectar::dec_max_rows(); ++R) {
    ++g_cases;
    const size_t s = nectar::dec_smem_for_rows(R);
    const int tile = nectar::dec_tile(R);
    CHECK(s <= kMaxSmemPerCta, "R %d smem %zu", R, s);
    // the K and V rings of 3 stages of tile rows of 256 bytes come first
    CHECK(s >= static_cast<size_t>(2) * 3 * tile * kD * 2, "R %d smem %zu below its ring", R, s);
    // 64-key tiles at up to 2 rows per warp are launch-bounded to 2 CTAs per SM
    const int rows_per_warp = R <= 2 ? R : (R <= 4 ? 2 : R);
    if (tile == 64 && rows_per_warp <= 2)
      CHECK(2 * (s + kReservedPerCta) <= kSmemPerSm, "R %d: two CTAs of %zu B do not fit", R, s);
  }
  return true;
}

// 64-bit linear congruential generator (Knuth's MMIX constants)
struct Lcg {
  uint64_t s;
  uint64_t next() { return s = s * 6364136223846793005ull + 1442695040888963407ull; }
  int64_t in(int64_t lo, int64_t hi) { return lo + static_cast<int64_t>((next() >> 11) % (hi - lo + 1)); }
};

}  // namespace

int main() {
  // workload shapes: (layers x KV heads, cached keys, query rows per KV head)
  const struct { int heads; int64_t n, rows; } shapes[] = {
      {28 * 8, 32768, 2},   {32 * 8, 131072, 4},  {32 * 8, 131072, 64},  {36 * 8, 4096, 4096},
      {28 * 4, 65536, 448}, {32 * 8, 131072, 1024}, {1, 1, 1},          {1, 128, 1},
      {1, 129, 8},          {2, 1000, 4},          {8, 65, 3},           {0, 4096, 2},
  };
  const int sm_counts[] = {148, 132, 1, 2, 7};
  for (const auto& w : shapes) {
    for (int sms : sm_counts) {
      for (int cps = 1; cps <= 2; ++cps)
        for (int tile : {64, 128})
          if (!check_decode(w.heads, w.n, sms, cps, tile)) return 1;
      if (w.heads > 0 && !check_tc(w.heads, w.n, w.rows, sms)) return 1;
    }
  }
  Lcg g{20241203};
  for (int i = 0; i < 4000; ++i) {
    const int heads = static_cast<int>(g.in(1, 320));
    const int64_t n = g.in(1, i % 4 == 0 ? 262144 : 5000);
    const int64_t rows = g.in(1, 5000);
    const int sms = static_cast<int>(g.in(1, 160));
    if (!check_decode(heads, n, sms, static_cast<int>(g.in(1, 2)), g.in(0, 1) ? 64 : 128)) return 1;
    if (!check_tc(heads, n, rows, sms)) return 1;
  }
  if (!check_smem()) return 1;
  std::printf("ok %lld\n", static_cast<long long>(g_cases));
  return 0;
}
