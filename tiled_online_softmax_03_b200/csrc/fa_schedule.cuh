// fa_schedule.cuh — work decomposition shared by the kernel and the host.
//
// The query side is cut into Q tiles of BM = 128 rows of one (b, hq). For one
// (b, hk) the G = Hq/Hk query heads of the group and the NM = ceil(N/128)
// m-blocks give G·NM tiles, listed by (m-block, head-in-group) and taken two at
// a time: a work unit is such a pair, so both tiles of a unit read the same
// K/V head (with G >= 2 they are two query heads at the same m-block — the
// head packing of the GQA page "深度探索Flash-Attention中GQA性能调优技术解析",
// section PackGQA — and with G = 1 they are two consecutive m-blocks).
//
// Causal problems list units heaviest first (largest m-block first, every
// (b, hk) at that level before the next level) so that a persistent grid that
// walks the list in a serpentine order ends with its lightest work.
//
// Split-KV (the num_splits setting of the GQA page "深度探索Flash-Attention中
// GQA性能调优技术解析"): with `splits` > 1 every unit above becomes `splits`
// consecutive units, each covering one contiguous chunk of the unit's K/V
// tiles; their partial results are merged afterwards by log-sum-exp.
#pragma once
#include <cstdint>

#ifdef __CUDACC__
#define FA_HD __host__ __device__ __forceinline__
#else
#define FA_HD inline
#endif

namespace fa {

constexpr int BM = 128;  // query rows per Q tile
constexpr int BN = 128;  // keys per K/V tile

struct Shape {
  int B, Hq, Hk, N, causal;
  int G;       // Hq / Hk
  int NM;      // m-blocks per head
  int NP;      // tile pairs per (b, hk)
  int splits;  // K/V chunks per tile pair (1 = no split)
  int num_units;
};

FA_HD Shape make_shape(int B, int Hq, int Hk, int N, int causal, int splits = 1) {
  Shape s;
  s.B = B; s.Hq = Hq; s.Hk = Hk; s.N = N; s.causal = causal ? 1 : 0;
  s.G = Hq / Hk;
  s.NM = (N + BM - 1) / BM;
  s.NP = (s.G * s.NM + 1) / 2;
  s.splits = splits < 1 ? 1 : splits;
  s.num_units = B * Hk * s.NP * s.splits;
  return s;
}

struct Unit {
  int b, hk;
  int hq[2], mb[2];
  int present[2];
  int split;    // K/V chunk of the tile pair (0 when not split)
  int key_len;  // valid keys of batch b, in [0, N]
  int j0;       // first K/V tile of the unit
  int n[2];     // one past the last K/V tile each Q tile visits (n[t] <= j0: none)
  int nmax;     // max(n[0], n[1], j0)
};

// Which Q tiles unit u holds (independent of key lengths).
FA_HD void decode_unit(const Shape& s, int u, Unit& U) {
  U.split = u % s.splits;
  u /= s.splits;
  const int bhk_count = s.B * s.Hk;
  int pair, bhk;
  if (s.causal) {
    pair = s.NP - 1 - u / bhk_count;
    bhk = u % bhk_count;
  } else {
    bhk = u / s.NP;
    pair = u % s.NP;
  }
  U.b = bhk / s.Hk;
  U.hk = bhk % s.Hk;
  for (int t = 0; t < 2; ++t) {
    const int x = 2 * pair + t;
    U.present[t] = x < s.G * s.NM;
    U.mb[t] = U.present[t] ? x / s.G : 0;
    U.hq[t] = U.hk * s.G + (U.present[t] ? x % s.G : 0);
  }
}

// K/V tile range once the batch's valid key count is known: all tiles a Q
// tile needs, or this split's contiguous share of the pair's range.
FA_HD void resolve_unit(const Shape& s, int key_len, Unit& U) {
  U.key_len = key_len;
  int full = 0;
  for (int t = 0; t < 2; ++t) {
    int kv_end = key_len;
    if (s.causal) {
      const int last_row_end = (U.mb[t] + 1) * BM;  // keys j <= i < (mb+1)·BM
      kv_end = kv_end < last_row_end ? kv_end : last_row_end;
    }
    U.n[t] = (U.present[t] && kv_end > 0) ? (kv_end + BN - 1) / BN : 0;
    full = U.n[t] > full ? U.n[t] : full;
  }
  const int chunk = (full + s.splits - 1) / s.splits;
  U.j0 = U.split * chunk < full ? U.split * chunk : full;
  const int jhi = U.j0 + chunk < full ? U.j0 + chunk : full;
  U.nmax = U.j0;
  for (int t = 0; t < 2; ++t) {
    U.n[t] = U.n[t] < jhi ? U.n[t] : jhi;
    if (U.n[t] < U.j0) U.n[t] = U.j0;
    U.nmax = U.n[t] > U.nmax ? U.n[t] : U.nmax;
  }
}

// Does Q tile t of the unit visit any K/V tile?
FA_HD bool tile_active(const Unit& U, int t) { return U.n[t] > U.j0; }

// Does K/V tile j need the element mask for Q tile t? (partial key tile, or
// the causal diagonal; tiles wholly above the diagonal are never visited)
FA_HD bool tile_needs_mask(const Shape& s, const Unit& U, int t, int j) {
  return (j + 1) * BN > U.key_len || (s.causal && j >= U.mb[t]);
}

// Serpentine assignment of units to the CTAs of a persistent grid.
FA_HD int unit_for(int cta, int it, int grid) {
  return it * grid + ((it & 1) ? grid - 1 - cta : cta);
}

}  // namespace fa
