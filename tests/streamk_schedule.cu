// Test helper (host program): walks the fused GEMM's stream-K schedule -- the kernel's own sk_units / sk_unit /
// sk_cta_of, compiled for the host -- over many (tiles, stages per tile, CTAs) and checks that it is a partition:
// every stage of every tile is done exactly once, a tile's parts come from consecutive CTAs in stage order with
// slabs z = 0, 1, ..., the part count equals what the reduction sums, the LoRA stages run once per tile (in slab
// 0), and every CTA gets floor or ceil of T / P stages.  Prints one line per case: "ok ..." or "FAIL ...".
// With the argument "planted" the last CTA walks the schedule of a grid one CTA larger (a plausible mistake: the
// grid size and the P the schedule assumes disagree); every case must then fail.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../qlora_fine_tuning_blockwise_b200/csrc/umma_gemm.cuh"

using namespace qlora;

static bool g_planted = false;

static bool check(int tiles, int S, int P, int n_extra) {
  UmmaArgs a{};
  a.tiles_i = tiles;
  a.sk_stages = S;
  a.n_extra = n_extra;
  const long long T = static_cast<long long>(tiles) * S;
  std::vector<int> done(T, 0), extra(tiles, 0), parts(tiles, 0), last_cta(tiles, -1), next_stage(tiles, 0);
  for (int c = 0; c < P; ++c) {
    long long work = 0;
    const long long Pc = (g_planted && c == P - 1) ? P + 1 : P;
    const int n = sk_units(a, c, Pc);
    for (int u = 0; u < n; ++u) {
      const Unit U = sk_unit(a, c, Pc, u);
      const int t = U.i0 / 128;
      if (t < 0 || t >= tiles || U.n_main <= 0 || U.main_begin != next_stage[t] || U.z != parts[t] ||
          (last_cta[t] >= 0 && last_cta[t] != c - 1)) {
        std::printf("FAIL tiles=%d S=%d P=%d: cta %d unit %d (tile %d begin %d n %d z %d)\n", tiles, S, P, c, u, t,
                    U.main_begin, U.n_main, U.z);
        return false;
      }
      for (int k = 0; k < U.n_main; ++k) done[static_cast<long long>(t) * S + U.main_begin + k] += 1;
      extra[t] += U.n_extra;
      if (U.n_extra > 0 && U.z != 0) {
        std::printf("FAIL tiles=%d S=%d P=%d: LoRA stages outside slab 0\n", tiles, S, P);
        return false;
      }
      next_stage[t] = U.main_begin + U.n_main;
      last_cta[t] = c;
      parts[t] += 1;
      work += U.n_main;
    }
    if (work != T / P && work != (T + P - 1) / P) {
      std::printf("FAIL tiles=%d S=%d P=%d: cta %d has %lld stages\n", tiles, S, P, c, work);
      return false;
    }
  }
  for (long long x = 0; x < T; ++x)
    if (done[x] != 1) {
      std::printf("FAIL tiles=%d S=%d P=%d: stage %lld done %d times\n", tiles, S, P, x, done[x]);
      return false;
    }
  for (int t = 0; t < tiles; ++t) {
    const long long n = sk_cta_of(static_cast<long long>(t) * S + S - 1, T, P) - sk_cta_of(static_cast<long long>(t) * S, T, P) + 1;
    if (n != parts[t] || next_stage[t] != S || extra[t] != n_extra) {
      std::printf("FAIL tiles=%d S=%d P=%d: tile %d parts %d (reduction sums %lld), extra %d\n", tiles, S, P, t,
                  parts[t], n, extra[t]);
      return false;
    }
  }
  std::printf("ok tiles=%d S=%d P=%d\n", tiles, S, P);
  return true;
}

int main(int argc, char** argv) {
  g_planted = argc > 1 && argv[1][0] == 'p';
  bool all = true;
  all &= check(224, 32, 148, 1);   // 16 tokens x 8192 -> 28672, four-block stages
  all &= check(8, 16, 32, 1);
  all &= check(17, 8, 34, 1);
  all &= check(1, 8, 2, 0);
  all &= check(1, 64, 16, 1);
  all &= check(148, 8, 148, 2);    // one tile per CTA
  all &= check(149, 8, 148, 1);
  all &= check(300, 5, 148, 1);
  std::srand(7);
  for (int i = 0; i < 300; ++i) {
    const int tiles = 1 + std::rand() % 400, S = 1 + std::rand() % 64;
    const long long T = static_cast<long long>(tiles) * S;
    const int P = 1 + static_cast<int>(std::rand() % (T < 148 ? T : 148));
    all &= check(tiles, S, P, std::rand() % 3);
  }
  if (g_planted) {  // every case must have failed
    return all ? 1 : 0;
  }
  return all ? 0 : 1;
}
