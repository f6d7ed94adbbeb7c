// fa_bwd_sm100.cuh — attention backward (dQ, dK, dV) for B200 (sm_100a).
// Included by fa_fwd_sm100.cu inside namespace fa (it shares the bounded
// waits, the PTX wrappers and the device status word of the forward).
//
// What it computes: the gradient of O = softmax(scale·QKᵀ + mask)·V for an
// upstream dO (page "FlashAttention 在昇腾 NPU 上是怎么省显存的？…": the v2
// kernel reworks the backward so that S and P need not be kept). P is rebuilt
// from Q, K and the forward's LSE:
//     P = exp(S − LSE),  dV = Pᵀ·dO,  dP = dO·Vᵀ,  D = rowsum(dO ⊙ O),
//     dS = P ⊙ (dP − D),  dQ = scale·dS·K,  dK = scale·dSᵀ·Q.
//
// Decomposition: a work unit is one 128-key block n of one (b, hk). Its dK and
// dV accumulate in tensor memory over every (query head of the group, query
// tile m) that sees the block — one "step" each — and are written once at the
// unit's end, so they need no atomics. dQ of a step is a partial sum over this
// key block only; it is added into an fp32 buffer by TMA reduce-add and
// scaled and rounded by a final kernel.
//
// Per step (Q, dO, LSE·log2e and D of query tile m staged by TMA, two stages):
//   MMA warp      Sᵀ = K·Qᵀ and dPᵀ = V·dOᵀ into TMEM (keys are the M rows)
//   softmax warps (eight: thread = key row, warps 0-3 queries 0-63 of the
//                 tile, warps 4-7 queries 64-127): Pᵀ = exp2(Sᵀ·scale·log2e −
//                 LSE·log2e) (masked keys → 0), dSᵀ = Pᵀ ⊙ (dPᵀ − D); Pᵀ and dSᵀ
//                 go to TMEM as 16-bit pairs over Sᵀ and dPᵀ, then dSᵀ (read back
//                 from TMEM) to shared memory in the 128-byte-swizzled layout
//                 of an MN-major operand
//   MMA warp      dV += Pᵀ·dO, dK += dSᵀ·Q (A from TMEM), dQ_part = dS·K
//                 (A = dSᵀ read MN-major from shared memory) into the dPᵀ
//                 columns
//   drain warps   thread = query row: dQ_part from TMEM into the dSᵀ tile
//                 (free once the dQ MMA has read it) as 32-column fp32 boxes,
//                 added into the fp32 dQ buffer by TMA reduce-add
// TMEM columns: Sᵀ/Pᵀ [0,128), dPᵀ/dSᵀ/dQ_part [128,256), dV and dK after;
// the 16-bit pairs of queries 64·h + [0, 64) occupy columns 64·h + [0, 32)
// of the Sᵀ and dPᵀ ranges.

namespace bwd {

constexpr int BK = 128;  // keys per unit
constexpr int BQ = 128;  // queries per step
constexpr int NUM_THREADS = 512;
constexpr int TMEM_COLS = 512;

enum {
  BB_KV_FULL = 0,   // TMA -> MMA: K and V of the unit loaded
  BB_KV_EMPTY = 1,  // MMA -> TMA: the unit's MMAs no longer read K, V
  BB_QD_FULL = 2,   // [2] TMA -> MMA, softmax: Q, dO, LSE·log2e, D of a step
  BB_QD_EMPTY = 4,  // [2] MMA (commit) + 8 softmax warps -> TMA: stage read
  BB_S_FULL = 6,    // MMA -> softmax: Sᵀ in TMEM
  BB_P_READY = 7,   // softmax -> MMA: Pᵀ, dSᵀ in TMEM and dSᵀ in smem
  BB_DQ_FULL = 8,   // MMA -> drain: dQ_part in TMEM
  BB_DQ_FREE = 9,   // drain -> MMA: dQ_part read
  BB_ACC_FULL = 10, // MMA -> drain: the unit's dK, dV complete
  BB_ACC_FREE = 11, // drain -> MMA: dK, dV read
  BB_DRAIN = 12,    // MMA drain on the abort path
  BB_STG_FREE = 13, // drain -> softmax: the dSᵀ tile, used as dQ staging, read by TMA
  BB_DP_FULL = 14,  // MMA -> softmax: dPᵀ in TMEM
  BB_COUNT = 15
};

// Shared memory, no slack: the tiles need a 1 KB-aligned base, which the
// kernel checks (and reports) instead of padding 1 KB it does not have at d=128.
template <int D>
struct BLayout {
  static constexpr int TILE = 128 * D * 2;          // one K, V, Q or dO tile
  static constexpr int OFF_BAR = 0;
  static constexpr int OFF_MISC = 128;              // tmem base, abort flag
  static constexpr int OFF_LD = 1024;               // [2 stages] LSE·log2e[128], D[128]
  static constexpr int OFF_K = 3072;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;        // [2 stages]
  static constexpr int OFF_DO = OFF_Q + 2 * TILE;   // [2 stages]
  static constexpr int OFF_DS = OFF_DO + 2 * TILE;  // dSᵀ [128 keys][128 queries], 2 boxes
  static constexpr int BYTES = OFF_DS + BK * BQ * 2;
  static_assert(OFF_K % 1024 == 0 && TILE % 1024 == 0, "tile alignment");
  static_assert(BYTES <= 232448, "shared memory budget");
};

struct BParams {
  int B, Hq, Hk, N, G, NM, Npad, causal, num_units;
  const int32_t* key_pad_lens;
  const float* lse2;  // [B·Hq][Npad] LSE·log2e; +inf for rows with no key and padding
  const float* dsum;  // [B·Hq][Npad] rowsum(dO ⊙ O); 0 in padding
  float* dqacc;       // [B·Hq][N][D] fp32 dQ/scale accumulator (zeroed)
  void* dk;           // [B·Hk][N][D] 16-bit
  void* dv;
  float scale_log2;   // scale·log2e
  float scale;
  unsigned long long timeout_ns;
  int ng;             // head groups of the unit order (0: one group)
};

struct BUnit {
  int b, hk, n, key_len, m_lo, nm, steps;
};

// Unit u: key block n = u / (B·Hk) (causal: smallest n, the most query tiles,
// first), (b, hk) = u % (B·Hk). Steps: every query head of the group × query
// tiles m >= m_lo (m_lo = n when causal); none if the block holds no valid key.
// With ng > 0 groups the (b, hk) heads are cut into ng near-equal groups and
// the order above runs within one group after the other, so that the CTAs in
// flight read the Q and dO tiles of a few heads, which stay in L2.
__device__ __forceinline__ bool bwd_unit(const BParams& p, int it, BUnit& U) {
  const int u = unit_for(blockIdx.x, it, gridDim.x);
  if (u >= p.num_units) return false;
  const int bhk_count = p.B * p.Hk;
  int bhk;
  if (p.ng > 0) {
    const int nkb = p.num_units / bhk_count;  // key blocks per head
    const int base = bhk_count / p.ng, rem = bhk_count % p.ng;
    const int big_units = (base + 1) * nkb;
    int g, r, gh;
    if (u < rem * big_units) {
      g = u / big_units;
      r = u - g * big_units;
      gh = base + 1;
    } else {
      const int v = u - rem * big_units;
      g = rem + v / (base * nkb);
      r = v - (g - rem) * base * nkb;
      gh = base;
    }
    U.n = r / gh;
    bhk = g * base + (g < rem ? g : rem) + r % gh;
  } else {
    U.n = u / bhk_count;
    bhk = u % bhk_count;
  }
  U.b = bhk / p.Hk;
  U.hk = bhk % p.Hk;
  int L = p.N;
  if (p.key_pad_lens != nullptr) {
    L = __ldg(p.key_pad_lens + U.b);
    L = L < 0 ? 0 : (L > p.N ? p.N : L);
  }
  U.key_len = L;
  U.m_lo = p.causal ? U.n : 0;
  U.nm = p.NM - U.m_lo;
  U.steps = (U.n * BK < L) ? p.G * U.nm : 0;
  return true;
}

__host__ __device__ constexpr uint32_t idesc_ab(bool bf16, int n, bool a_mn, bool b_mn) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ uint32_t bbar(uint32_t sbase, int i) { return sbase + 8 * i; }

// ------------------------------------------------------------------ loader
template <int D>
__device__ void bwd_load(const BParams& p, uint32_t sbase, const Ctl& c, const CUtensorMap* tm_q,
                         const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                         const CUtensorMap* tm_do) {
  using L = BLayout<D>;
  int units = 0, step_ct = 0;
  bool ok = true, kv_armed = false;
  uint32_t kv_last = 0, qd_armed = 0, qd_last[2] = {0, 0};
  BUnit U;
  for (int it = 0; ok && bwd_unit(p, it, U); ++it) {
    if (U.steps == 0) continue;
    if (units > 0 && !(ok = wait_bar(bbar(sbase, BB_KV_EMPTY), (units - 1) & 1, c))) break;
    const uint32_t kvf = bbar(sbase, BB_KV_FULL);
    mbar_arrive_expect_tx(kvf, 2 * L::TILE);
    kv_last = units & 1;
    kv_armed = true;
    const int kv_head = U.b * p.Hk + U.hk;
    for (int bx = 0; bx < D / 64; ++bx) {
      tma_load_3d(sbase + L::OFF_K + bx * SW128_BOX_BYTES, tm_k, bx * 64, U.n * BK, kv_head, kvf);
      tma_load_3d(sbase + L::OFF_V + bx * SW128_BOX_BYTES, tm_v, bx * 64, U.n * BK, kv_head, kvf);
    }
    ++units;
    for (int s = 0; s < U.steps && ok; ++s, ++step_ct) {
      const int stg = step_ct & 1, use = step_ct >> 1;
      if (use > 0 && !(ok = wait_bar(bbar(sbase, BB_QD_EMPTY + stg), (use - 1) & 1, c))) break;
      const uint32_t full = bbar(sbase, BB_QD_FULL + stg);
      mbar_arrive_expect_tx(full, 2 * L::TILE + 1024);
      qd_last[stg] = use & 1;
      qd_armed |= 1u << stg;
      const int hq = U.hk * p.G + s / U.nm, m = U.m_lo + s % U.nm;
      const int head = U.b * p.Hq + hq;
      for (int bx = 0; bx < D / 64; ++bx) {
        tma_load_3d(sbase + L::OFF_Q + stg * L::TILE + bx * SW128_BOX_BYTES, tm_q, bx * 64, m * BQ,
                    head, full);
        tma_load_3d(sbase + L::OFF_DO + stg * L::TILE + bx * SW128_BOX_BYTES, tm_do, bx * 64,
                    m * BQ, head, full);
      }
      const size_t row0 = (size_t)head * p.Npad + (size_t)m * BQ;
      bulk_load_1d(sbase + L::OFF_LD + stg * 1024, p.lse2 + row0, 512, full);
      bulk_load_1d(sbase + L::OFF_LD + stg * 1024 + 512, p.dsum + row0, 512, full);
    }
  }
  if (!ok) {
    // Let every armed copy land before the CTA can exit (bounded, short).
    volatile int no_abort = 0;
    Ctl drain{&no_abort, 100000000ull};
    if (kv_armed) wait_bar(bbar(sbase, BB_KV_FULL), kv_last, drain);
    for (int s = 0; s < 2; ++s)
      if (qd_armed >> s & 1) wait_bar(bbar(sbase, BB_QD_FULL + s), qd_last[s], drain);
  }
}

// --------------------------------------------------------------------- MMA
template <int D, bool BF16>
__device__ void bwd_mma(const BParams& p, uint32_t sbase, uint32_t tmem, const Ctl& c) {
  using L = BLayout<D>;
  constexpr uint32_t ID_S = idesc_ab(BF16, BQ, false, false);  // Sᵀ, dPᵀ: both K-major
  constexpr uint32_t ID_G = idesc_ab(BF16, D, false, true);    // dV, dK: A in TMEM, B MN-major
  constexpr uint32_t ID_Q = idesc_ab(BF16, D, true, true);     // dQ: A and B MN-major
  const uint32_t t_s = tmem, t_dp = tmem + 128, t_dv = tmem + 256, t_dk = tmem + 256 + D;
  const uint64_t k_kmaj = sdesc(sbase + L::OFF_K, 16, 1024);
  const uint64_t v_kmaj = sdesc(sbase + L::OFF_V, 16, 1024);
  const uint64_t k_mn = sdesc(sbase + L::OFF_K, SW128_BOX_BYTES, 1024);
  const uint64_t ds_mn = sdesc(sbase + L::OFF_DS, SW128_BOX_BYTES, 1024);
  // C[128 keys][128 queries] = A[keys][d]·B[queries][d]ᵀ, both K-major (d contiguous)
  auto mma_kk = [&](uint32_t d_t, uint64_t a, uint64_t b) {
    umma_ss_warp(d_t, a, b, ID_S, 0u);
#pragma unroll
    for (int k = 1; k < D / 16; ++k) {
      const uint32_t off = ((k >> 2) * SW128_BOX_BYTES + (k & 3) * 32) >> 4;
      umma_ss_warp(d_t, a + off, b + off, ID_S, 1u);
    }
  };
  // C[128][D] (+)= A(TMEM, 16-bit pairs)[128][128]·B[128][D], B MN-major. The
  // pairs of queries 64·h + [0, 64) sit in columns 64·h + [0, 32) (the softmax
  // halves' layout), so K step k (16 queries) reads columns 64·(k/4) + 8·(k%4).
  auto mma_tk = [&](uint32_t d_t, uint32_t a_t, uint64_t b, uint32_t acc) {
    umma_ts_warp(d_t, a_t, b, ID_G, acc);
#pragma unroll
    for (int k = 1; k < BQ / 16; ++k)
      umma_ts_warp(d_t, a_t + (k >> 2) * 64 + (k & 3) * 8, b + ((k * 16 * 128) >> 4), ID_G, 1u);
  };
  int units = 0, acc_units = 0, step_ct = 0;
  bool ok = true;
  BUnit U;
  for (int it = 0; ok && bwd_unit(p, it, U); ++it) {
    if (U.steps == 0) continue;
    if (!(ok = wait_bar_warp(bbar(sbase, BB_KV_FULL), units & 1, c))) break;
    ++units;
    for (int s = 0; s < U.steps && ok; ++s, ++step_ct) {
      const int stg = step_ct & 1, use = step_ct >> 1;
      if (!(ok = wait_bar_warp(bbar(sbase, BB_QD_FULL + stg), use & 1, c))) break;
      tc_fence_after();
      const uint32_t q_base = sbase + L::OFF_Q + stg * L::TILE;
      const uint32_t do_base = sbase + L::OFF_DO + stg * L::TILE;
      mma_kk(t_s, k_kmaj, sdesc(q_base, 16, 1024));                      // Sᵀ = K·Qᵀ
      umma_commit_warp(bbar(sbase, BB_S_FULL));
      // dPᵀ overwrites the previous step's dQ_part: wait for the drain
      if (step_ct > 0 && !(ok = wait_bar_warp(bbar(sbase, BB_DQ_FREE), (step_ct - 1) & 1, c)))
        break;
      tc_fence_after();
      mma_kk(t_dp, v_kmaj, sdesc(do_base, 16, 1024));                    // dPᵀ = V·dOᵀ
      umma_commit_warp(bbar(sbase, BB_DP_FULL));
      if (!(ok = wait_bar_warp(bbar(sbase, BB_P_READY), step_ct & 1, c))) break;
      if (s == 0 && acc_units > 0 &&
          !(ok = wait_bar_warp(bbar(sbase, BB_ACC_FREE), (acc_units - 1) & 1, c)))
        break;
      tc_fence_after();
      const uint32_t acc = s > 0 ? 1u : 0u;
      mma_tk(t_dv, t_s, sdesc(do_base, SW128_BOX_BYTES, 1024), acc);     // dV += Pᵀ·dO
      mma_tk(t_dk, t_dp, sdesc(q_base, SW128_BOX_BYTES, 1024), acc);     // dK += dSᵀ·Q
      // dQ_part = dS·K over this block's 128 keys (16 keys per MMA)
      umma_ss_warp(t_dp, ds_mn, k_mn, ID_Q, 0u);
#pragma unroll
      for (int k = 1; k < BK / 16; ++k) {
        const uint32_t off = (k * 16 * 128) >> 4;
        umma_ss_warp(t_dp, ds_mn + off, k_mn + off, ID_Q, 1u);
      }
      umma_commit_warp(bbar(sbase, BB_DQ_FULL));
      umma_commit_warp(bbar(sbase, BB_QD_EMPTY + stg));
    }
    if (!ok) break;
    umma_commit_warp(bbar(sbase, BB_ACC_FULL));
    umma_commit_warp(bbar(sbase, BB_KV_EMPTY));
    ++acc_units;
  }
  if (!ok) {
    volatile int no_abort = 0;
    Ctl drain{&no_abort, 100000000ull};
    umma_commit_warp(bbar(sbase, BB_DRAIN));
    wait_bar_warp(bbar(sbase, BB_DRAIN), 0, drain);
  }
}

// ----------------------------------------------------------------- softmax
template <int D, bool BF16>
__device__ void bwd_softmax(const BParams& p, uint8_t* smem, uint32_t sbase, uint32_t tmem,
                            const Ctl& c) {
  using L = BLayout<D>;
  const int k = threadIdx.x & 127;       // key row of the block = TMEM lane
  const int half = (threadIdx.x >> 7) & 1;  // queries [64·half, 64·half + 64) of the tile
  const uint32_t lane_base = (uint32_t)((threadIdx.x >> 5) & 3) * 32;
  const uint32_t t_s = tmem + (lane_base << 16), t_dp = t_s + 128;
  uint8_t* ds_row = smem + L::OFF_DS + half * SW128_BOX_BYTES + k * 128;
  const int sw = k & 7;
  int step_ct = 0;
  BUnit U;
  for (int it = 0; bwd_unit(p, it, U); ++it) {
    if (U.steps == 0) continue;
    const int key = U.n * BK + k;
    const bool key_ok = key < U.key_len;
    for (int s = 0; s < U.steps; ++s, ++step_ct) {
      const int stg = step_ct & 1, use = step_ct >> 1;
      if (!wait_bar_warp(bbar(sbase, BB_QD_FULL + stg), use & 1, c)) return;
      if (!wait_bar_warp(bbar(sbase, BB_S_FULL), step_ct & 1, c)) return;
      tc_fence_after();
      const int m = U.m_lo + s % U.nm;
      const float* lse2 = reinterpret_cast<const float*>(smem + L::OFF_LD + stg * 1024);
      const float* dsum = lse2 + 128;
      // queries j of the tile with key <= m·128 + j (causal), all if not causal
      const int q_first = p.causal ? key - m * BQ : 0;
      // phase 1 (while the tensor core computes dPᵀ): P for this thread's 64
      // queries, kept in fp32 for dS, and written to TMEM as 16-bit pairs
      float pf[64];
      // every query of this thread's half allowed (off the causal diagonal)?
      const bool all_ok = key_ok && q_first <= 64 * half;
#pragma unroll
      for (int cq = 0; cq < 2; ++cq) {
        const int cc = 2 * half + cq;  // 32-query chunk of the tile
        uint32_t sv[32];
        tmem_ld_x32(t_s + 32 * cc, sv);
        tmem_wait_ld();
        reg_pin_x32(sv);
        uint32_t pk[16];
        const float4* l4 = reinterpret_cast<const float4*>(lse2 + 32 * cc);
        if (all_ok) {
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 l = l4[g];
            const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              pf[32 * cq + 4 * g + e] =
                  ex2_approx(fmaf(__uint_as_float(sv[4 * g + e]), p.scale_log2, -lv[e]));
          }
        } else {
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            const float4 l = l4[g];
            const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 32 * cc + 4 * g + e;
              const float x = fmaf(__uint_as_float(sv[4 * g + e]), p.scale_log2, -lv[e]);
              pf[32 * cq + 4 * g + e] = (key_ok && j >= q_first) ? ex2_approx(x) : 0.f;
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = round_pack<BF16>(pf[32 * cq + 2 * i], pf[32 * cq + 2 * i + 1]);
        // packed pairs of half h go to columns 64·h + [0, 32): only columns this
        // thread has already read, never the other half's unread ones
        tmem_st_x16(t_s + 64 * half + 16 * cq, pk);
      }
      // phase 2: dS = P ⊙ (dP − D)
      if (!wait_bar_warp(bbar(sbase, BB_DP_FULL), step_ct & 1, c)) return;
      tc_fence_after();
#pragma unroll
      for (int cq = 0; cq < 2; ++cq) {
        const int cc = 2 * half + cq;
        uint32_t dp[32];
        tmem_ld_x32(t_dp + 32 * cc, dp);
        tmem_wait_ld();
        reg_pin_x32(dp);
        uint32_t dk2[16];
        const float4* d4 = reinterpret_cast<const float4*>(dsum + 32 * cc);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float4 dd = d4[g];
          const int i = 4 * g;
          dk2[2 * g] = round_pack<BF16>(pf[32 * cq + i] * (__uint_as_float(dp[i]) - dd.x),
                                        pf[32 * cq + i + 1] * (__uint_as_float(dp[i + 1]) - dd.y));
          dk2[2 * g + 1] = round_pack<BF16>(pf[32 * cq + i + 2] * (__uint_as_float(dp[i + 2]) - dd.z),
                                            pf[32 * cq + i + 3] * (__uint_as_float(dp[i + 3]) - dd.w));
        }
        tmem_st_x16(t_dp + 64 * half + 16 * cq, dk2);
      }
      tmem_wait_st();
      // dSᵀ to the shared tile (it doubles as the drain's dQ staging: wait until
      // TMA has read that): this thread's 64 queries are one 128-byte row of box
      // `half`, 16-byte chunk i stored at chunk i ^ (k & 7)
      if (step_ct > 0 && !wait_bar_warp(bbar(sbase, BB_STG_FREE), (step_ct - 1) & 1, c)) return;
      uint32_t w[32];
      tmem_ld_x32(t_dp + 64 * half, w);
      tmem_wait_ld();
      reg_pin_x32(w);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        *reinterpret_cast<uint4*>(ds_row + ((i ^ sw) << 4)) =
            make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      fence_proxy_async_smem();  // generic-proxy writes of dSᵀ, read by the MMA
      tc_fence_before();
      mbar_arrive(bbar(sbase, BB_P_READY));
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bbar(sbase, BB_QD_EMPTY + stg));
    }
  }
}

// --------------------------------------------------- dQ drain and dK/dV out
template <int D, bool BF16>
__device__ void bwd_drain(const BParams& p, uint8_t* smem, uint32_t sbase, uint32_t tmem,
                          const Ctl& c, const CUtensorMap* tm_dq) {
  using L = BLayout<D>;
  const int r = threadIdx.x & 127;  // TMEM lane: query row (dQ_part), key row (dK, dV)
  const uint32_t lane_base = (uint32_t)((threadIdx.x >> 5) & 3) * 32;
  const uint32_t t_row = tmem + (lane_base << 16);
  const int lane = threadIdx.x & 31, wl = (threadIdx.x >> 5) & 3;
  constexpr int STG_BOX = BQ * 32 * 4;  // one [128 rows][32 fp32] staging box, 16 KB
  int step_ct = 0, acc_units = 0;
  BUnit U;
  for (int it = 0; bwd_unit(p, it, U); ++it) {
    for (int s = 0; s < U.steps; ++s, ++step_ct) {
      if (!wait_bar_warp(bbar(sbase, BB_DQ_FULL), step_ct & 1, c)) goto done;
      tc_fence_after();
      const int hq = U.hk * p.G + s / U.nm, m = U.m_lo + s % U.nm;
      const int head = U.b * p.Hq + hq;
      // dQ_part through the 32 KB dSᵀ tile: two staging boxes of [128 rows][32
      // fp32]; each warp stages its own 32 rows and its lane 0 adds that 4 KB
      // slab into dQ by TMA (no cross-warp barrier). Row r, 16-byte chunk i
      // sits at chunk i ^ (r & 7) of its 128-byte row (128-byte swizzle). All
      // TMEM reads come before any wait on TMA, so the MMA warp gets the
      // columns back (DQ_FREE) as early as possible.
      auto stage = [&](const uint32_t* v, int box, int cc) {
        const uint32_t slab = L::OFF_DS + box * STG_BOX + wl * 32 * 128;
        uint8_t* row = smem + slab + (r & 31) * 128;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          *reinterpret_cast<uint4*>(row + ((i ^ (r & 7)) << 4)) =
              make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tma_reduce_add_3d(tm_dq, sbase + slab, 32 * cc, m * BQ + wl * 32, head);
      };
      uint32_t v[D / 32][32];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld_x32(t_row + 128 + 32 * cc, v[cc]);
      tmem_wait_ld();
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) reg_pin_x32(v[cc]);
      tc_fence_before();
      mbar_arrive(bbar(sbase, BB_DQ_FREE));
#pragma unroll
      for (int pair = 0; pair < D / 64; ++pair) {
        if (pair > 0) {  // the previous pair's staging read by TMA?
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
        }
        stage(v[2 * pair], 0, 2 * pair);
        stage(v[2 * pair + 1], 1, 2 * pair + 1);
        if (lane == 0) bulk_commit_group();
      }
      if (lane == 0) {
        bulk_wait_group_read<0>();
        mbar_arrive(bbar(sbase, BB_STG_FREE));
      }
      __syncwarp();
    }
    // ---- the unit's dK (×scale) and dV rows
    const int key = U.n * BK + r;
    const size_t orow = ((size_t)(U.b * p.Hk + U.hk) * p.N + key) * D;
    const bool has = U.steps > 0;
    if (has) {
      if (!wait_bar_warp(bbar(sbase, BB_ACC_FULL), acc_units & 1, c)) goto done;
      tc_fence_after();
    }
#pragma unroll 1
    for (int which = 0; which < 2; ++which) {  // 0: dV, 1: dK
      uint16_t* out = reinterpret_cast<uint16_t*>(which ? p.dk : p.dv) + orow;
      const float mul = which ? p.scale : 1.f;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        if (has) {
          tmem_ld_x32(t_row + 256 + which * D + 32 * cc, v);
          tmem_wait_ld();
          reg_pin_x32(v);
          if (which == 1 && cc == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bbar(sbase, BB_ACC_FREE));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        if (key < p.N) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = cvt2<D, BF16>(__uint_as_float(v[8 * i]) * mul, __uint_as_float(v[8 * i + 1]) * mul);
            w.y = cvt2<D, BF16>(__uint_as_float(v[8 * i + 2]) * mul, __uint_as_float(v[8 * i + 3]) * mul);
            w.z = cvt2<D, BF16>(__uint_as_float(v[8 * i + 4]) * mul, __uint_as_float(v[8 * i + 5]) * mul);
            w.w = cvt2<D, BF16>(__uint_as_float(v[8 * i + 6]) * mul, __uint_as_float(v[8 * i + 7]) * mul);
            *reinterpret_cast<uint4*>(out + 32 * cc + 8 * i) = w;
          }
        }
      }
    }
    if (has) ++acc_units;
  }
done:
  // the TMA reductions into dQ complete before the CTA may exit
  if (lane == 0) bulk_wait_group<0>();
  __syncwarp();
}

template <int D, bool BF16>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, const BParams p) {
  using L = BLayout<D>;
  extern __shared__ __align__(1024) uint8_t bsmem[];
  const uint32_t sbase = smem_addr(bsmem);
  if (sbase & 1023) {  // the layout has no room to realign; report and stop
    if (threadIdx.x == 0) atomicCAS(&g_fa_status, 0, (int)FA_ERR_UNSUPPORTED);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bsmem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bsmem + L::OFF_MISC + 4);
  if (threadIdx.x == 0) {
    mbar_init(bbar(sbase, BB_KV_FULL), 1);
    mbar_init(bbar(sbase, BB_KV_EMPTY), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bbar(sbase, BB_QD_FULL + s), 1);
      mbar_init(bbar(sbase, BB_QD_EMPTY + s), 1 + 8);  // MMA commit + one per softmax warp
    }
    mbar_init(bbar(sbase, BB_S_FULL), 1);
    mbar_init(bbar(sbase, BB_DP_FULL), 1);
    mbar_init(bbar(sbase, BB_P_READY), 256);
    mbar_init(bbar(sbase, BB_DQ_FULL), 1);
    mbar_init(bbar(sbase, BB_DQ_FREE), 128);
    mbar_init(bbar(sbase, BB_ACC_FULL), 1);
    mbar_init(bbar(sbase, BB_ACC_FREE), 128);
    mbar_init(bbar(sbase, BB_DRAIN), 1);
    mbar_init(bbar(sbase, BB_STG_FREE), 4);  // lane 0 of each drain warp
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 12) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 13 && lane == 0) {
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
    tma_prefetch_map(&tm_do);
    tma_prefetch_map(&tm_dq);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Ctl ctl{abort_flag, p.timeout_ns};
  // Register split: 2×136 (softmax) + 144 (drain: a whole dQ_part row in
  // registers) + 96 (MMA, loads) = 4 × 128.
  if (warp < 8) {
    setmaxnreg_inc<136>();
    bwd_softmax<D, BF16>(p, bsmem, sbase, tmem, ctl);
  } else if (warp < 12) {
    setmaxnreg_inc<144>();
    bwd_drain<D, BF16>(p, bsmem, sbase, tmem, ctl, &tm_dq);
  } else {
    setmaxnreg_dec<96>();
    if (warp == 12) bwd_mma<D, BF16>(p, sbase, tmem, ctl);
    if (warp == 13 && lane == 0) bwd_load<D>(p, sbase, ctl, &tm_q, &tm_k, &tm_v, &tm_do);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// D_i = Σ_c dO_ic·O_ic and LSE·log2e per padded row (+inf where the forward
// found no key, and in padding rows i >= N); zeroes the dQ accumulator rows.
// One warp per row.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_pre_kernel(const void* __restrict__ o,
                                                         const void* __restrict__ dout,
                                                         const float* __restrict__ lse,
                                                         float* lse2, float* dsum, float* dqacc,
                                                         long long BH, int N, int Npad) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long rows = BH * Npad;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < rows;
       row += nwarps) {
    const long long bh = row / Npad;
    const int i = (int)(row % Npad);
    if (i < N) {
      const size_t src = ((size_t)bh * N + i) * D + lane * E;
      const uint16_t* po = reinterpret_cast<const uint16_t*>(o) + src;
      const uint16_t* pd = reinterpret_cast<const uint16_t*>(dout) + src;
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float a, b;
        if constexpr (BF16) {
          a = __uint_as_float((uint32_t)po[e] << 16);
          b = __uint_as_float((uint32_t)pd[e] << 16);
        } else {
          a = __half2float(__ushort_as_half(po[e]));
          b = __half2float(__ushort_as_half(pd[e]));
        }
        acc = fmaf(a, b, acc);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      float* z = dqacc + ((size_t)bh * N + i) * D + lane * E;
#pragma unroll
      for (int e = 0; e < E; ++e) z[e] = 0.f;
      if (lane == 0) {
        const float l = lse[(size_t)bh * N + i];
        dsum[row] = acc;
        lse2[row] = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
      }
    } else if (lane == 0) {
      dsum[row] = 0.f;
      lse2[row] = INFINITY;
    }
  }
}

// dQ = scale · (fp32 accumulator), rounded to the 16-bit type; 8 elements per thread.
template <bool BF16>
__global__ void __launch_bounds__(256) fa_bwd_post_kernel(const float* __restrict__ dqacc,
                                                          void* dq, float scale, long long n8) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(dqacc) + 2 * i);
    const float4 b = __ldg(reinterpret_cast<const float4*>(dqacc) + 2 * i + 1);
    uint4 w;
    w.x = cvt2<64, BF16>(a.x * scale, a.y * scale);
    w.y = cvt2<64, BF16>(a.z * scale, a.w * scale);
    w.z = cvt2<64, BF16>(b.x * scale, b.y * scale);
    w.w = cvt2<64, BF16>(b.z * scale, b.w * scale);
    reinterpret_cast<uint4*>(dq)[i] = w;
  }
}

}  // namespace bwd
