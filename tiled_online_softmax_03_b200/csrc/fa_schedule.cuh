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
// walks the list in a serpentine order ends with its lightest work. When the
// grid would have fewer than ~12 CTAs on each (b, hk) head at a time, the
// heads are cut into `ng` near-equal groups and that order runs within one
// group after the other, so that the CTAs in flight share each head's K/V
// tiles in L2; each group is then dealt out to the CTAs by itself.
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
  int ng;      // causal: groups of (b, hk) heads in the unit order (0 = one group)
  int num_units;
  int gw[2], gr[2];  // grouped order: full waves and units left over, in a group of
                     // one head more (0) and in the others (1), for the launch's grid
};

FA_HD Shape make_shape(int B, int Hq, int Hk, int N, int causal, int splits = 1, int ng = 0) {
  Shape s;
  s.B = B; s.Hq = Hq; s.Hk = Hk; s.N = N; s.causal = causal ? 1 : 0;
  s.G = Hq / Hk;
  s.NM = (N + BM - 1) / BM;
  s.NP = (s.G * s.NM + 1) / 2;
  s.splits = splits < 1 ? 1 : splits;
  s.ng = (causal && ng > 1 && ng <= B * Hk) ? ng : 0;
  s.num_units = B * Hk * s.NP * s.splits;
  s.gw[0] = s.gw[1] = s.gr[0] = s.gr[1] = 0;
  return s;
}

// Records the waves of each group size for a `grid`-CTA launch of the grouped order.
FA_HD void set_group_grid(Shape& s, int grid) {
  if (s.ng == 0 || grid < 1) return;
  const int small = (s.B * s.Hk / s.ng) * s.NP * s.splits;
  const int sizes[2] = {small + s.NP * s.splits, small};
  for (int i = 0; i < 2; ++i) {
    s.gw[i] = sizes[i] / grid;
    s.gr[i] = sizes[i] - s.gw[i] * grid;
  }
}

// Head groups for a causal problem on a `grid`-CTA launch (0: one group):
// about 12 CTAs per (b, hk) head at a time, only when fewer are in flight
// without groups, when the K and V of all heads (kv_head_bytes each) would
// not stay in half of the L2 but those of one group would, and for problems
// of at least eight waves of units, each group at least four waves.
inline int group_count(int B, int Hq, int Hk, int N, int causal, int grid, long long kv_head_bytes,
                       long long l2_bytes) {
  if (!causal || grid < 1 || B < 1 || Hk < 1 || Hq % Hk != 0) return 0;
  const long long heads = (long long)B * Hk;
  const long long np = ((long long)(Hq / Hk) * ((N + BM - 1) / BM) + 1) / 2;
  const long long per_group = grid / 12 > 0 ? grid / 12 : 1;
  if (heads * np < 8LL * grid || heads <= per_group) return 0;
  if (2 * heads * kv_head_bytes <= l2_bytes || 2 * per_group * kv_head_bytes > l2_bytes) return 0;
  long long ng = (heads + per_group - 1) / per_group;
  const long long min_heads = (4LL * grid + np - 1) / np;
  if (ng > heads / min_heads) ng = heads / min_heads;
  return ng > 1 ? (int)ng : 0;
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

// Which Q tiles unit u holds (independent of key lengths). GROUPED = false
// leaves out the head-grouped order (for code that never runs it).
template <bool GROUPED = true>
FA_HD void decode_unit(const Shape& s, int u, Unit& U) {
  U.split = u % s.splits;
  u /= s.splits;
  const int bhk_count = s.B * s.Hk;
  int pair, bhk;
  if (GROUPED && s.causal && s.ng > 0) {
    // groups of base + 1 heads first (rem of them), then groups of base heads
    const int base = bhk_count / s.ng, rem = bhk_count % s.ng;
    const int big_units = (base + 1) * s.NP;
    int g, r, gh;
    if (u < rem * big_units) {
      g = u / big_units;
      r = u - g * big_units;
      gh = base + 1;
    } else {
      const int v = u - rem * big_units;
      g = rem + v / (base * s.NP);
      r = v - (g - rem) * base * s.NP;
      gh = base;
    }
    pair = s.NP - 1 - r / gh;
    bhk = g * base + (g < rem ? g : rem) + r % gh;
  } else if (s.causal) {
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

// The same under the head-grouped order (s.ng > 0): the serpentine walk starts
// afresh in every group, so each group is shared out evenly by itself (its
// lightest units last), and a CTA done with one group goes on to the next.
// Needs set_group_grid(s, grid). Returns s.num_units once the CTA has no unit left.
FA_HD int unit_for_grouped(const Shape& s, int cta, int it, int grid) {
  const int rem = s.B * s.Hk % s.ng;  // the first rem groups hold one head more
  int off = 0;
  for (int g = 0; g < s.ng; ++g) {
    // iterations CTA `cta` takes in this group: full waves, and maybe one of the last
    const int w = g < rem ? s.gw[0] : s.gw[1], r = g < rem ? s.gr[0] : s.gr[1];
    const int n = w + (((w & 1) ? grid - 1 - cta : cta) < r);
    if (it < n) return off + unit_for(cta, it, grid);
    it -= n;
    off += w * grid + r;
  }
  return s.num_units;
}

}  // namespace fa
