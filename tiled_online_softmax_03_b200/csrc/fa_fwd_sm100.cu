// fa_fwd_sm100.cu — exact attention forward for B200 (sm_100a) and its C ABI.
//
// What it computes: O = softmax(scale·QKᵀ + mask)·V and LSE per query row
// (page "FlashAttention (VI)", section "Vấn đề của cơ chế attention tiêu
// chuẩn"), tile by tile with the online-softmax recurrence of the page "MCU 上
// Transformer 模型的 Flash Attention 实现在 256KB SRAM 约束下的分块计算与内存建模
// 方案", §二: per query row a running max m, a running denominator l and an
// unnormalised O, rescaled by exp(m_old − m_new) when m grows, divided by l once
// at the end (§三). Scores never leave the SM: S lives in tensor memory (TMEM),
// P overwrites it there, only O and LSE are written to HBM.
//
// One persistent CTA per SM (512 threads, one 512-column TMEM allocation)
// walks work units of two 128-row Q tiles that share a K/V head
// (fa_schedule.cuh). Warp roles:
//   warps 0-3   softmax for Q tile 0 (thread r owns row r: TMEM lane r)
//   warps 4-7   softmax for Q tile 1
//   warps 8-11  correction (rescale O in TMEM at d = 128 with 16-bit inputs)
//               and epilogue (O/l, LSE, stores)
//   warp 12     tcgen05.mma issue (one thread)
//   warp 13     TMA loads (one thread)
//   warps 14-15 bias mode: TMA loads of the bias tiles of Q tile 0 / 1
//                (one thread each); otherwise no work
// Per K/V tile j and Q tile t the MMA thread issues S_t = Q_t·K_jᵀ into TMEM,
// the softmax warps turn S_t into P_t (16-bit, written over S_t in TMEM) and
// the running statistics, O_t is rescaled when a row's reference max moved
// (by the correction warps, or by the softmax warps themselves at d = 64 and
// in FP8), and the MMA thread issues O_t += P_t·V_j with P read from TMEM. The two Q tiles alternate, so
// the tensor core works on one tile while the other tile's softmax runs.
//
// Pipelines use mbarriers; every wait is bounded (globaltimer) and a wait that
// runs out records FA_ERR_DEVICE_TIMEOUT in g_fa_status instead of hanging.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/fa.h"
#include "fa_ptx.cuh"
#include "fa_schedule.cuh"

namespace fa {

__device__ int g_fa_status;  // first device-side error of any launch (0 = none)

constexpr int NUM_THREADS = 512;

constexpr int TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: keep a stale max until it is 2^8 behind
constexpr int SW128_BOX_BYTES = BM * 128;  // one 128-row box of 64 16-bit columns
constexpr int OST_BYTES = 32 * 32 * 2;     // one 32-row × 32-column output staging box

// TMEM columns: S/P for tile 0 and 1, then O. At d = 128 the four regions
// fill the 512 columns.
//
// Short-sequence configuration (d = 64): units hold only a few K/V tiles, so
// the unit boundary matters as much as the steady state. There the Q tiles
// and O are double-buffered (a unit's Q tiles load during the previous unit;
// its first P·V does not wait for the previous unit's epilogue to read O
// out: TMEM has 128 spare columns), units are decoded once into a ring of
// records in shared memory, and the MMA warp issues the next unit's first S
// right behind each tile's last P·V.
__device__ constexpr uint32_t S_COL[2] = {0, 128};
template <int D>
struct TmemO {
  static constexpr bool SHORT = D == 64;
  static constexpr int BUFS = SHORT ? 2 : 1;  // O buffers per tile
  // final-statistics buffers per tile: a unit's softmax may finish while the
  // epilogues of the BUFS units before it are still pending
  static constexpr int NSTATS = SHORT ? 4 : 2;
  __host__ __device__ static constexpr uint32_t col(int t, int buf) { return 256 + (t + 2 * buf) * D; }
};

constexpr int UNIT_RING = 4;
constexpr int OFF_URING = 576;  // [UNIT_RING] × 64 bytes, after the barriers

// Barrier slots.
enum {
  BAR_QFULL = 0,    // [2 tiles][2 Q buffers] TMA -> MMA: Q tile loaded
  BAR_QEMPTY = 4,   // [2 tiles][2 Q buffers] MMA -> TMA: the unit's last QK no longer needs it
  BAR_SFULL = 8,    // [2] MMA -> softmax: S tile ready in TMEM
  BAR_PFULL = 10,   // [2] softmax -> MMA: P written to TMEM
  BAR_AFULL = 12,   // [2] softmax -> correction: rescale factors in smem (d = 128 bf16/fp16)
  BAR_OCORR = 14,   // [2] correction -> MMA: O rescaled (d = 128 bf16/fp16)
  BAR_PVDONE = 16,  // [2 tiles][2 O buffers] MMA -> epilogue: last P·V of the unit done
  BAR_OFREE = 20,   // [2 tiles][2 O buffers] epilogue -> MMA: O read out of TMEM
  BAR_STATS = 24,   // [2 tiles][4 buffers] softmax -> epilogue: final m, l in smem
  BAR_DRAIN = 32,   // MMA drain on the abort path
  BAR_PHALF = 33,   // [2] softmax -> MMA: P of the first 64 keys written to TMEM
  BAR_BFULL = 35,   // [2] TMA -> softmax: bias tile loaded (bias mode)
  BAR_BEMPTY = 37,  // [2] softmax -> TMA: bias tile read
  BAR_UFULL = 39,   // [UNIT_RING] producer -> every role: unit record written (d = 64)
  BAR_UEMPTY = 43,  // [UNIT_RING] every role -> producer: unit record read (d = 64)
  BAR_KV = 47       // [STAGES] full, then [STAGES] empty
};

// Shared memory: barriers and flags first, then 1 KB-aligned tiles. With an
// additive bias the K/V ring is halved to make room for one 128×128 16-bit
// bias tile per Q tile.
// MODE: 0 = plain, 1 = additive bias, 2 = FP8 (E4M3 Q, K, V), 3 = plain with
// the head-grouped unit order (a kernel of its own, so that the others carry
// no code for it).
template <int D, int MODE = 0>
struct Layout {
  static constexpr bool BIAS = MODE == 1, FP8 = MODE == 2, GROUPED = MODE == 3;
  static constexpr int ELEM = FP8 ? 1 : 2;  // bytes per Q, K, V element
  static constexpr bool RING = TmemO<D>::SHORT;  // unit ring, early next-unit S
  // Who rescales O when a row's reference max moves: the softmax warps
  // themselves, before signalling half of P (d = 64 and FP8, measured faster),
  // or the correction warps, which the MMA warp then waits for (d = 128 with
  // 16-bit inputs: faster where rescales are frequent, as with peaked rows).
  static constexpr bool SELF_RESCALE = TmemO<D>::SHORT || MODE == 2;
  static constexpr int QBUF = TmemO<D>::SHORT ? 2 : 1;
  static constexpr int Q_BYTES = BM * D * ELEM;
  static constexpr int KV_BYTES = BN * D * ELEM;
  static constexpr int STAGES = BIAS ? ((D == 128) ? 2 : 4) : ((D == 128 && !FP8) ? 4 : 8);
  static constexpr int BIAS_BYTES = BIAS ? BM * BN * 2 : 0;
  static constexpr int NUM_BARS = BAR_KV + 2 * STAGES;
  static constexpr int OFF_BAR = 0;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;     // tmem base, abort flag
  static constexpr int OFF_Q = 1024;
  static constexpr int OFF_KV = OFF_Q + 2 * QBUF * Q_BYTES;  // Q: [QBUF][2 tiles]
  static constexpr int OFF_BIAS = OFF_KV + STAGES * KV_BYTES;  // [2 tiles] bias mode only
  static constexpr int OFF_OST = OFF_BIAS + 2 * BIAS_BYTES;
  static constexpr int OFF_ALPHA = OFF_OST + 8 * OST_BYTES;   // [2 tiles][128] float
  static constexpr int OFF_STATS = OFF_ALPHA + 2 * BM * 4;    // [NSTATS buf][2 tiles][128] float4
  static constexpr int BYTES = OFF_STATS + TmemO<D>::NSTATS * 2 * BM * 16;
  static constexpr int ALLOC = BYTES + 1024;                  // base is rounded up to 1 KB
  static_assert(OFF_MISC + 16 <= OFF_URING && OFF_URING + UNIT_RING * 64 <= OFF_Q, "barrier area");
  static_assert(OFF_KV % 1024 == 0 && OFF_BIAS % 1024 == 0 && OFF_OST % 1024 == 0,
                "tile alignment");
  static_assert(ALLOC <= 232448, "shared memory budget");
};

struct Params {
  const int32_t* key_pad_lens;
  float* lse;
  float* o_part;    // split-KV: [splits][B·Hq][N][d] fp32 partial O (normalised), else null
  float* lse_part;  // split-KV: [splits][B·Hq][N] fp32 partial LSE
  float o_scale;    // FP8 mode: the V descale, applied to O in the epilogue
  int bias_bmul;    // bias mode: bias plane of (b, hq) is (b·bias_bmul)·bias_H + hq·bias_hmul
  int bias_hmul;
  int bias_H;
  Shape s;
  float scale_log2;
  unsigned long long timeout_ns;
};

// ------------------------------------------------------------ descriptors
// UMMA shared-memory descriptor, sm_100 format: start address >> 4 in bits
// 0-13, leading byte offset >> 4 in 16-29, stride byte offset >> 4 in 32-45,
// version 1 in bit 46, layout (2 = 128-byte swizzle) in bits 61-63.
__host__ __device__ constexpr uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFF) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor for kind::f16 with fp32 accumulation, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(bool bf16, int n, bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// High word of every shared-memory descriptor used here (1024-byte stride
// byte offset, version 1, 128-byte swizzle); only the low word varies.
constexpr uint32_t SDESC_HI = (uint32_t)(sdesc(0, 16, 1024) >> 32);
// Two spellings of the same MMAs: full 64-bit descriptors, or their low words
// with SDESC_HI as a constant (fewer live registers in the issuing warp).
template <bool F8>
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  if constexpr (F8) umma_ss_f8_warp(d, a, b, id, acc);
  else umma_ss_warp(d, a, b, id, acc);
}
template <bool F8>
__device__ __forceinline__ void mma_ss(uint32_t d, uint32_t a, uint32_t b, uint32_t id, uint32_t acc) {
  umma_ss_lo<F8, SDESC_HI, SDESC_HI>(d, a, b, id, acc);
}
template <bool F8>
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id, uint32_t acc) {
  if constexpr (F8) umma_ts_f8_warp(d, a_tmem, b, id, acc);
  else umma_ts_warp(d, a_tmem, b, id, acc);
}
template <bool F8>
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint32_t b, uint32_t id, uint32_t acc) {
  umma_ts_lo<F8, SDESC_HI>(d, a_tmem, b, id, acc);
}

// ------------------------------------------------------------ bounded waits
struct Ctl {
  volatile int* abort_flag;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, const Ctl& c) {
  const uint64_t t0 = global_timer_ns();
  while (true) {
    // Sleep in the barrier (up to 0.2 ms per try) rather than spin: waiting
    // warps share issue slots with the softmax warps on the same SMSP.
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if (*c.abort_flag) return false;
    if (global_timer_ns() - t0 > c.timeout_ns) {
      *c.abort_flag = 1;
      atomicCAS(&g_fa_status, 0, (int)FA_ERR_DEVICE_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const Ctl& c) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, c);
}
// Warp-uniform form for roles whose later instructions are warp-collective.
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, const Ctl& c) {
  const bool ok = wait_bar(bar, parity, c);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ uint32_t bar_addr(uint32_t sbase, int i) {
  return sbase + 8 * i;  // barriers sit at the start of shared memory in every layout
}

__device__ __forceinline__ int key_len_of(const Params& p, int b) {
  if (p.key_pad_lens == nullptr) return p.s.N;
  int l = __ldg(p.key_pad_lens + b);
  return l < 0 ? 0 : (l > p.s.N ? p.s.N : l);
}

// Unit `it` of this CTA (serpentine order, by head group in the grouped
// kernel), decoded; false past the last one.
template <bool GROUPED>
__device__ __forceinline__ bool next_unit(const Params& p, int it, Unit& U) {
  const int u = GROUPED ? unit_for_grouped(p.s, blockIdx.x, it, gridDim.x)
                        : unit_for(blockIdx.x, it, gridDim.x);
  if (u >= p.s.num_units) return false;
  decode_unit<GROUPED>(p.s, u, U);
  resolve_unit(p.s, key_len_of(p, U.b), U);
  return true;
}

// Unit records: 16 ints, {valid, b, hk, split, hq0, hq1, mb0, mb1, present0,
// present1, key_len, j0, n0, n1, nmax, -}; valid = 0 ends the walk.
__device__ __forceinline__ void write_unit(uint8_t* smem, int slot, const Unit& U, int valid) {
  int4* d = reinterpret_cast<int4*>(smem + OFF_URING + slot * 64);
  d[0] = make_int4(valid, U.b, U.hk, U.split);
  d[1] = make_int4(U.hq[0], U.hq[1], U.mb[0], U.mb[1]);
  d[2] = make_int4(U.present[0], U.present[1], U.key_len, U.j0);
  d[3] = make_int4(U.n[0], U.n[1], U.nmax, 0);
}
__device__ __forceinline__ int read_unit(const uint8_t* smem, int slot, Unit& U) {
  const int4* r = reinterpret_cast<const int4*>(smem + OFF_URING + slot * 64);
  const int4 a = r[0], b = r[1], c = r[2], d = r[3];
  U.b = a.y; U.hk = a.z; U.split = a.w;
  U.hq[0] = b.x; U.hq[1] = b.y; U.mb[0] = b.z; U.mb[1] = b.w;
  U.present[0] = c.x; U.present[1] = c.y; U.key_len = c.z; U.j0 = c.w;
  U.n[0] = d.x; U.n[1] = d.y; U.nmax = d.z;
  return a.x;
}
// Record `it` for a whole warp: wait until it is written, copy it, release
// the slot (one arrival per warp). 1: a unit, 0: no more units, -1: the wait
// gave up.
__device__ __forceinline__ int take_unit_warp(const uint8_t* smem, uint32_t sbase, int it,
                                              const Ctl& c, Unit& U) {
  const int slot = it & (UNIT_RING - 1);
  if (!wait_bar_warp(bar_addr(sbase, BAR_UFULL + slot), (it / UNIT_RING) & 1, c)) return -1;
  const int valid = read_unit(smem, slot, U);
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar_addr(sbase, BAR_UEMPTY + slot));
  return valid;
}
// Unit `it` for a role: from the unit ring (RING), else decoded here.
template <bool RING, bool GROUPED>
__device__ __forceinline__ int get_unit_warp(const Params& p, const uint8_t* smem, uint32_t sbase,
                                             int it, const Ctl& c, Unit& U) {
  if constexpr (RING) return take_unit_warp(smem, sbase, it, c, U);
  else return next_unit<GROUPED>(p, it, U) ? 1 : 0;
}
// The same for a role run by one thread.
__device__ __forceinline__ int take_unit(const uint8_t* smem, uint32_t sbase, int it, const Ctl& c,
                                         Unit& U) {
  const int slot = it & (UNIT_RING - 1);
  if (!wait_bar(bar_addr(sbase, BAR_UFULL + slot), (it / UNIT_RING) & 1, c)) return -1;
  const int valid = read_unit(smem, slot, U);
  mbar_arrive(bar_addr(sbase, BAR_UEMPTY + slot));
  return valid;
}
template <bool RING, bool GROUPED>
__device__ __forceinline__ int get_unit(const Params& p, const uint8_t* smem, uint32_t sbase, int it,
                                        const Ctl& c, Unit& U) {
  if constexpr (RING) return take_unit(smem, sbase, it, c, U);
  else return next_unit<GROUPED>(p, it, U) ? 1 : 0;
}

// ============================================================ TMA producer
// One thread. Loads each unit's Q tiles and streams its K/V tiles through
// the ring of stages. With the unit ring (d = 64) it also decodes each unit
// and publishes it there before its loads, so every role sees the next unit
// early. Q tile t of the k-th unit that uses it goes to Q buffer k mod QBUF.
template <int D, int MODE>
__device__ void role_load(const Params& p, uint8_t* smem, uint32_t sbase, const Ctl& c,
                          const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v) {
  using L = Layout<D, MODE>;
  constexpr bool FP8 = L::FP8;
  constexpr int QBUF = L::QBUF;
  (void)FP8;
  uint32_t qe_ph = 0;     // one bit per (tile, Q buffer)
  int qcnt[2] = {0, 0};   // units that used each tile so far
  int st = 0;
  uint32_t kv_ph = 0;
  // parity of the last arming of each barrier, for the abort drain
  uint32_t armed_q = 0, armed_kv = 0, last_q_ph = 0, last_kv_ph[L::STAGES];
  bool ok = true;
  Unit U;
  for (int it = 0; ok; ++it) {
    const bool valid = next_unit<L::GROUPED>(p, it, U);
    if constexpr (L::RING) {
      const int slot = it & (UNIT_RING - 1);
      if (!(ok = wait_bar(bar_addr(sbase, BAR_UEMPTY + slot), ((it / UNIT_RING) & 1) ^ 1, c))) break;
      write_unit(smem, slot, U, valid ? 1 : 0);
      mbar_arrive(bar_addr(sbase, BAR_UFULL + slot));
    }
    if (!valid) break;
    for (int t = 0; t < 2 && ok; ++t) {
      if (!tile_active(U, t)) continue;
      const int qb = qcnt[t]++ & (QBUF - 1), qi = 2 * t + qb;
      if (!(ok = wait_bar(bar_addr(sbase, BAR_QEMPTY + qi), ((qe_ph >> qi) & 1) ^ 1, c))) break;
      qe_ph ^= 1u << qi;
      const uint32_t full = bar_addr(sbase, BAR_QFULL + qi);
      mbar_arrive_expect_tx(full, L::Q_BYTES);
      last_q_ph = (armed_q >> qi & 1) ? last_q_ph ^ (1u << qi) : last_q_ph & ~(1u << qi);
      armed_q |= 1u << qi;
      const int head = U.b * p.s.Hq + U.hq[t];
      // a 128-byte-wide box: 64 16-bit or 128 8-bit columns
      constexpr int BOX_COLS = 128 / L::ELEM;
      for (int bx = 0; bx < D / BOX_COLS; ++bx)
        tma_load_3d(sbase + L::OFF_Q + (qb * 2 + t) * L::Q_BYTES + bx * SW128_BOX_BYTES, tm_q,
                    bx * BOX_COLS, U.mb[t] * BM, head, full);
    }
    const int kv_head = U.b * p.s.Hk + U.hk;
    for (int j = U.j0; j < U.nmax && ok; ++j) {
      for (int which = 0; which < 2; ++which) {  // K_j then V_j
        if (!(ok = wait_bar(bar_addr(sbase, BAR_KV + L::STAGES + st), kv_ph ^ 1, c))) break;
        const uint32_t full = bar_addr(sbase, BAR_KV + st);
        mbar_arrive_expect_tx(full, L::KV_BYTES);
        last_kv_ph[st] = kv_ph;
        armed_kv |= 1u << st;
        if constexpr (FP8) {
          // K_j: [128 keys][128 8-bit d] one box. V_j from the transposed copy
          // Vᵀ [d][N]: d rows × keys j·128 .. +127 (K-major for the P·V product).
          if (which)
            tma_load_3d(sbase + L::OFF_KV + st * L::KV_BYTES, tm_v, j * BN, 0, kv_head, full);
          else
            tma_load_3d(sbase + L::OFF_KV + st * L::KV_BYTES, tm_k, 0, j * BN, kv_head, full);
        } else {
          const CUtensorMap* map = which ? tm_v : tm_k;
          for (int bx = 0; bx < D / 64; ++bx)
            tma_load_3d(sbase + L::OFF_KV + st * L::KV_BYTES + bx * SW128_BOX_BYTES, map, bx * 64,
                        j * BN, kv_head, full);
        }
        if (++st == L::STAGES) {
          st = 0;
          kv_ph ^= 1;
        }
      }
    }
  }
  if (!ok) {
    // Let every armed copy land before the CTA can exit (bounded, short).
    Ctl drain{c.abort_flag, 100000000ull};
    volatile int no_abort = 0;
    drain.abort_flag = &no_abort;
    for (int qi = 0; qi < 4; ++qi)
      if (armed_q >> qi & 1) wait_bar(bar_addr(sbase, BAR_QFULL + qi), (last_q_ph >> qi) & 1, drain);
    for (int s = 0; s < L::STAGES; ++s)
      if (armed_kv >> s & 1) wait_bar(bar_addr(sbase, BAR_KV + s), last_kv_ph[s], drain);
  }
}

// ============================================================= MMA issuer
// Bias tiles for Q tile t (bias mode; one thread each of warps 14 and 15):
// for every K/V tile j the tile visits, the 128×128 block of the bias plane
// at rows of the Q tile and keys of K/V tile j, as two 64-column boxes with
// the 128-byte swizzle, into the tile's single bias buffer. Rows and keys
// past N read as zero (they are masked or never stored).
template <int D>
__device__ void role_bias_load(const Params& p, const uint8_t* smem, uint32_t sbase, const Ctl& c,
                               const CUtensorMap* tm_b, int t) {
  using L = Layout<D, 1>;
  uint32_t be_ph = 0, last_ph = 0;
  bool armed = false, ok = true;
  Unit U;
  for (int it = 0; ok; ++it) {
    const int r = get_unit<Layout<D, 1>::RING, false>(p, smem, sbase, it, c, U);
    if (r <= 0) {
      ok = r == 0;
      break;
    }
    if (!tile_active(U, t)) continue;
    const int plane = U.b * p.bias_bmul * p.bias_H + U.hq[t] * p.bias_hmul;
    for (int j = U.j0; j < U.n[t] && ok; ++j) {
      if (!(ok = wait_bar(bar_addr(sbase, BAR_BEMPTY + t), be_ph ^ 1, c))) break;
      be_ph ^= 1;
      const uint32_t full = bar_addr(sbase, BAR_BFULL + t);
      mbar_arrive_expect_tx(full, L::BIAS_BYTES);
      last_ph = armed ? last_ph ^ 1 : 0;
      armed = true;
      for (int bx = 0; bx < BN / 64; ++bx)
        tma_load_3d(sbase + L::OFF_BIAS + t * L::BIAS_BYTES + bx * SW128_BOX_BYTES, tm_b,
                    j * BN + bx * 64, U.mb[t] * BM, plane, full);
    }
  }
  if (!ok && armed) {
    // Let the armed copy land before the CTA can exit (bounded, short).
    volatile int no_abort = 0;
    Ctl drain{&no_abort, 100000000ull};
    wait_bar(bar_addr(sbase, BAR_BFULL + t), last_ph, drain);
  }
}

// Short-sequence form of the MMA warp (d = 64; see role_mma for the rest).
// Per unit: S_t = Q_t·K_j0ᵀ for both tiles, then for every K/V tile j and
// tile t: O_t += P_t·V_j (in two 64-key halves, the first as soon as the
// softmax has stored half of P), then S_t for K_{j+1}. At a unit's last K/V
// tile the first S of the NEXT unit (with work) is issued right behind each
// tile's last P·V, so that tile's softmax restarts without waiting for the
// other tile or for the epilogue: the next unit's K_j0 follows this unit's
// last V_j in the ring of stages, its Q tiles were loaded into the other Q
// buffers during this unit, and its P·V goes to the other O buffers.
template <int D, bool BF16, int MODE>
__device__ void role_mma_lookahead(const Params& p, const uint8_t* smem, uint32_t sbase,
                                   uint32_t tmem, const Ctl& c) {
  using L = Layout<D, MODE>;
  constexpr bool FP8 = L::FP8;
  static_assert(TmemO<D>::BUFS == 2 && L::QBUF == 2, "the look-ahead form double-buffers Q and O");
  (void)FP8;
  // S = Q·Kᵀ, both K-major; O += P·V with V MN-major (16-bit) or, for FP8, Vᵀ
  // K-major (E4M3 is format 0 of kind::f8f6f4, as fp16 is of kind::f16)
  constexpr uint32_t IDESC_QK = idesc_f16(BF16 && !FP8, BN, false);
  constexpr uint32_t IDESC_PV = idesc_f16(BF16 && !FP8, D, !FP8);
  int st = 0;
  uint32_t kv_ph = 0;
  bool ok = true;

  // Issue cost matters as much as tensor time here: one 128x128x16 MMA runs
  // in ~64 cycles, so each issue must be a handful of instructions. The K
  // loops are unrolled with compile-time offsets added to a descriptor built
  // once per call (a K step adds its byte offset >> 4 to the start-address
  // field, bits 0-13, with no carry out since shared memory is < 256 KB), and
  // the accumulate flag is a compile-time constant except on the first step.
  // The plain kernels keep only the descriptors' low words live: the 64-bit
  // form spilled in this 80-register warp and ran 4-5 % slower. The bias and
  // FP8 kernels keep the 64-bit form (no spill in FP8; in the bias kernel the
  // low-word form timed 13 % slower).
  using Desc = std::conditional_t<MODE == 0 || MODE == 3, uint32_t, uint64_t>;
  const Desc q_desc0 = (Desc)sdesc(sbase + L::OFF_Q, 16, 1024);
  const Desc kv_desc0 = (Desc)sdesc(sbase + L::OFF_KV, 16, 1024);
  const Desc v_desc0 = FP8 ? kv_desc0 : (Desc)sdesc(sbase + L::OFF_KV, SW128_BOX_BYTES, 1024);
  auto issue_qk = [&](int t, int kst, int qb) {
    const Desc qd = q_desc0 + (Desc)(((qb * 2 + t) * L::Q_BYTES) >> 4);
    const Desc kd = kv_desc0 + (Desc)((kst * L::KV_BYTES) >> 4);
    const uint32_t d_s = tmem + S_COL[t];
    if constexpr (FP8) {  // K = 32 bytes per MMA, all inside one 128-byte row
      mma_ss<true>(d_s, qd, kd, IDESC_QK, 0u);
#pragma unroll
      for (int k = 1; k < D / 32; ++k) mma_ss<true>(d_s, qd + 2 * k, kd + 2 * k, IDESC_QK, 1u);
      return;
    }
    if constexpr (MODE == 0) {  // four MMAs per asm block (plain kernel; measured on the
                                // grouped kernel without gain, which keeps one per block)
      static_assert(D == 64 || D == 128, "head dim");
      umma_ss_lo_x4<SDESC_HI, SDESC_HI, 2, 2>(d_s, qd, kd, IDESC_QK, 0u);
      if constexpr (D == 128)
        umma_ss_lo_x4<SDESC_HI, SDESC_HI, 2, 2>(d_s, qd + (SW128_BOX_BYTES >> 4),
                                                 kd + (SW128_BOX_BYTES >> 4), IDESC_QK, 1u);
      return;
    }
    mma_ss<false>(d_s, qd, kd, IDESC_QK, 0u);
#pragma unroll
    for (int k = 1; k < D / 16; ++k) {
      const uint32_t off = ((k >> 2) * SW128_BOX_BYTES + (k & 3) * 32) >> 4;
      mma_ss<false>(d_s, qd + off, kd + off, IDESC_QK, 1u);
    }
  };
  // P·V over keys [64·h, 64·h + 64) of the tile (h = 0: first half, 1: second)
  // into the O buffer at TMEM column o_col.
  auto issue_pv_half = [&](int t, int vst, int h, uint32_t acc, uint32_t o_col) {
    // P: 16 keys = 8 TMEM columns (two 16-bit values per column); V: 16 key
    // rows of 128 bytes in each 64-column box, boxes SW128_BOX_BYTES apart.
    const Desc vd = v_desc0 + (Desc)((vst * L::KV_BYTES) >> 4);
    const uint32_t d_o = tmem + o_col;
    const uint32_t a_p = tmem + S_COL[t];
    if constexpr (FP8) {
      // P: 32 keys = 8 TMEM columns (four E4M3 values per column); Vᵀ rows
      // hold keys, 32 keys = 32 bytes of each 128-byte row
#pragma unroll
      for (int k = 2 * h; k < 2 * h + 2; ++k)
        mma_ts<true>(d_o, a_p + k * 8, vd + 2 * k, IDESC_PV, k == 0 ? acc : 1u);
      return;
    }
    const int k0 = h * (BN / 32);
    if constexpr (MODE == 0) {  // one asm block (plain kernel)
      umma_ts_lo_x4<SDESC_HI, 8, 128>(d_o, a_p + k0 * 8, vd + k0 * 128, IDESC_PV, acc);
      return;
    }
    mma_ts<false>(d_o, a_p + k0 * 8, vd + ((k0 * 16 * 128) >> 4), IDESC_PV, acc);
#pragma unroll
    for (int k = k0 + 1; k < k0 + BN / 32; ++k)
      mma_ts<false>(d_o, a_p + k * 8, vd + ((k * 16 * 128) >> 4), IDESC_PV, 1u);
  };

  // Phase bits, one per barrier the MMA warp waits on; QF and OF: one per
  // (tile, buffer).
  constexpr uint32_t QF = 0, PF = 4, PH = 8, OF = 10;
  uint32_t ph = 0;
  auto wait_flip = [&](int bar, uint32_t bit, uint32_t invert) {
    const bool r = wait_bar_warp(bar_addr(sbase, bar), ((ph >> bit) & 1u) ^ invert, c);
    ph ^= 1u << bit;
    return r;
  };
  // The MMA warp needs only the K/V ranges of a unit (tile t visits
  // [j0, n_t); units without work are skipped, so max(n0, n1) > j0).
  struct Range {
    int j0, n0, n1;
  };
  int it = 0;
  // Next unit with work (units whose tiles see no key are skipped: nothing
  // is loaded for them). 1: found, 0: none left, -1: a wait gave up.
  auto next_work = [&](Range& R) -> int {
    while (true) {
      Unit U;
      const int r = take_unit_warp(smem, sbase, it++, c, U);
      if (r <= 0) return r;
      if (U.nmax > U.j0) {
        R = Range{U.j0, U.n[0], U.n[1]};
        return 1;
      }
    }
  };
  // Buffer parities, one bit per tile: bits 0-1 the Q buffer the next unit
  // using the tile takes, 2-3 the current unit's Q buffers, 4-5 the next
  // unit's, 6-7 the current unit's O buffers. Q tile t of the k-th unit that
  // uses it sits in Q buffer k mod 2; O likewise.
  uint32_t bufs = 0;
  // First S of tile t of a unit from the K stage kst (already waited for),
  // from Q buffer q.
  auto first_s = [&](const Range& R, int t, int kst, int q) {
    const int qi = 2 * t + q;
    if (!wait_flip(BAR_QFULL + qi, QF + qi, 0)) return false;
    tc_fence_after();
    issue_qk(t, kst, q);
    umma_commit_warp(bar_addr(sbase, BAR_SFULL + t));
    if ((t ? R.n1 : R.n0) == R.j0 + 1) umma_commit_warp(bar_addr(sbase, BAR_QEMPTY + qi));
    return true;
  };
  // Takes the next Q buffer of tile t: returns it, records it as the
  // current (cur) or next unit's buffer, and flips the tile's parity.
  auto take_q = [&](int t, bool cur) {
    const int q = (bufs >> t) & 1;
    const int sh = (cur ? 2 : 4) + t;
    bufs = (bufs & ~(1u << sh)) | ((uint32_t)q << sh);
    bufs ^= 1u << t;
    return q;
  };

  Range U;
  int r0 = next_work(U);
  ok = r0 >= 0;
  bool have = r0 > 0;
  if (ok && have) {
    const int k0 = st;
    const uint32_t k0_ph = kv_ph;
    if (++st == L::STAGES) { st = 0; kv_ph ^= 1; }
    ok = wait_bar_warp(bar_addr(sbase, BAR_KV + k0), k0_ph, c);
    if (ok) tc_fence_after();
    for (int t = 0; t < 2 && ok; ++t)
      if ((t ? U.n1 : U.n0) > U.j0) ok = first_s(U, t, k0, take_q(t, true));
    if (ok) umma_commit_warp(bar_addr(sbase, BAR_KV + L::STAGES + k0));
  }
  while (ok && have) {
    const int j0 = U.j0, nmax = U.n0 > U.n1 ? U.n0 : U.n1;
    Range Un{0, 0, 0};
    bool have_next = false;
    for (int j = j0; j < nmax && ok; ++j) {
      const int vs = st;
      const uint32_t vs_ph = kv_ph;
      if (++st == L::STAGES) { st = 0; kv_ph ^= 1; }
      const bool last = j + 1 == nmax;
      if (last) {
        const int r = next_work(Un);
        ok = r >= 0;
        if (!ok) break;
        have_next = r > 0;
      }
      // K stage of this unit's next tile, or of the next unit's first tile
      int kn = -1;
      uint32_t kn_ph = 0;
      if (!last || have_next) {
        kn = st;
        kn_ph = kv_ph;
        if (++st == L::STAGES) { st = 0; kv_ph ^= 1; }
      }
      if (!(ok = wait_bar_warp(bar_addr(sbase, BAR_KV + vs), vs_ph, c))) break;
      bool kn_ready = false;
      auto need_kn = [&]() {
        if (kn_ready) return true;
        kn_ready = true;
        const bool r = wait_bar_warp(bar_addr(sbase, BAR_KV + kn), kn_ph, c);
        tc_fence_after();
        return r;
      };
      for (int t = 0; t < 2; ++t) {
        const int nt = t ? U.n1 : U.n0;
        const int ob = (bufs >> (6 + t)) & 1, qb = (bufs >> (2 + t)) & 1;
        if (j < nt) {
          if (!(ok = wait_flip(BAR_PHALF + t, PH + t, 0))) break;
          if (j == j0 && !(ok = wait_flip(BAR_OFREE + 2 * t + ob, OF + 2 * t + ob, 1))) break;
          tc_fence_after();
          const uint32_t o_col = TmemO<D>::col(t, ob);
          issue_pv_half(t, vs, 0, j > j0 ? 1u : 0u, o_col);
          if (!(ok = wait_flip(BAR_PFULL + t, PF + t, 0))) break;
          tc_fence_after();
          issue_pv_half(t, vs, 1, 1u, o_col);
          if (j == nt - 1) {
            umma_commit_warp(bar_addr(sbase, BAR_PVDONE + 2 * t + ob));
          } else {
            if (!(ok = need_kn())) break;
            issue_qk(t, kn, qb);
            umma_commit_warp(bar_addr(sbase, BAR_SFULL + t));
            if (j + 2 == nt) umma_commit_warp(bar_addr(sbase, BAR_QEMPTY + 2 * t + qb));
          }
        }
        if (last && have_next && (t ? Un.n1 : Un.n0) > Un.j0) {
          // the next unit's first S for this tile, right behind its last P·V
          // (its Q tile loaded into the other Q buffer during this unit)
          if (!(ok = need_kn())) break;
          if (!(ok = first_s(Un, t, kn, take_q(t, false)))) break;
        }
      }
      if (!ok) break;
      umma_commit_warp(bar_addr(sbase, BAR_KV + L::STAGES + vs));
      if (kn >= 0) umma_commit_warp(bar_addr(sbase, BAR_KV + L::STAGES + kn));
    }
    // this unit's tiles move to their other O buffer; the next unit's Q
    // buffers become the current ones
    bufs ^= (U.n0 > j0 ? 1u << 6 : 0u) | (U.n1 > j0 ? 1u << 7 : 0u);
    bufs = (bufs & ~(3u << 2)) | (((bufs >> 4) & 3u) << 2);
    U = Un;
    have = have_next;
  }
  if (!ok) {
    // Let every issued MMA finish before TMEM is released.
    volatile int no_abort = 0;
    Ctl drain{&no_abort, 100000000ull};
    umma_commit_warp(bar_addr(sbase, BAR_DRAIN));
    wait_bar_warp(bar_addr(sbase, BAR_DRAIN), 0, drain);
  }
}

// Run by the whole of warp 12, converged; one elected lane issues each
// tcgen05 instruction. Per unit: S_t = Q_t·K_j0ᵀ for both tiles, then for
// every K/V tile j and tile t: O_t += P_t·V_j (in two 64-key halves, the
// first as soon as the softmax has stored half of P), then S_t for K_{j+1}.
template <int D, bool BF16, int MODE>
__device__ void role_mma(const Params& p, const uint8_t* smem, uint32_t sbase, uint32_t tmem,
                         const Ctl& c) {
  using L = Layout<D, MODE>;
  constexpr bool FP8 = L::FP8;
  (void)FP8;
  if constexpr (L::RING) {
    role_mma_lookahead<D, BF16, MODE>(p, smem, sbase, tmem, c);
    return;
  }
  // S = Q·Kᵀ, both K-major; O += P·V with V MN-major (16-bit) or, for FP8, Vᵀ
  // K-major (E4M3 is format 0 of kind::f8f6f4, as fp16 is of kind::f16)
  constexpr uint32_t IDESC_QK = idesc_f16(BF16 && !FP8, BN, false);
  constexpr uint32_t IDESC_PV = idesc_f16(BF16 && !FP8, D, !FP8);
  int st = 0;
  uint32_t kv_ph = 0;
  bool ok = true;

  // Issue cost matters as much as tensor time here: one 128x128x16 MMA runs
  // in ~64 cycles, so each issue must be a handful of instructions. The K
  // loops are unrolled with compile-time offsets added to a descriptor built
  // once per call (a K step adds its byte offset >> 4 to the start-address
  // field, bits 0-13, with no carry out since shared memory is < 256 KB), and
  // the accumulate flag is a compile-time constant except on the first step.
  // The plain kernels keep only the descriptors' low words live: the 64-bit
  // form spilled in this 80-register warp and ran 4-5 % slower. The bias and
  // FP8 kernels keep the 64-bit form (no spill in FP8; in the bias kernel the
  // low-word form timed 13 % slower).
  using Desc = std::conditional_t<MODE == 0 || MODE == 3, uint32_t, uint64_t>;
  const Desc q_desc0 = (Desc)sdesc(sbase + L::OFF_Q, 16, 1024);
  const Desc kv_desc0 = (Desc)sdesc(sbase + L::OFF_KV, 16, 1024);
  const Desc v_desc0 = FP8 ? kv_desc0 : (Desc)sdesc(sbase + L::OFF_KV, SW128_BOX_BYTES, 1024);
  auto issue_qk = [&](int t, int kst) {
    const Desc qd = q_desc0 + (Desc)((t * L::Q_BYTES) >> 4);
    const Desc kd = kv_desc0 + (Desc)((kst * L::KV_BYTES) >> 4);
    const uint32_t d_s = tmem + S_COL[t];
    if constexpr (FP8) {  // K = 32 bytes per MMA, all inside one 128-byte row
      mma_ss<true>(d_s, qd, kd, IDESC_QK, 0u);
#pragma unroll
      for (int k = 1; k < D / 32; ++k) mma_ss<true>(d_s, qd + 2 * k, kd + 2 * k, IDESC_QK, 1u);
      return;
    }
    if constexpr (MODE == 0) {  // four MMAs per asm block (plain kernel; measured on the
                                // grouped kernel without gain, which keeps one per block)
      static_assert(D == 64 || D == 128, "head dim");
      umma_ss_lo_x4<SDESC_HI, SDESC_HI, 2, 2>(d_s, qd, kd, IDESC_QK, 0u);
      if constexpr (D == 128)
        umma_ss_lo_x4<SDESC_HI, SDESC_HI, 2, 2>(d_s, qd + (SW128_BOX_BYTES >> 4),
                                                 kd + (SW128_BOX_BYTES >> 4), IDESC_QK, 1u);
      return;
    }
    mma_ss<false>(d_s, qd, kd, IDESC_QK, 0u);
#pragma unroll
    for (int k = 1; k < D / 16; ++k) {
      const uint32_t off = ((k >> 2) * SW128_BOX_BYTES + (k & 3) * 32) >> 4;
      mma_ss<false>(d_s, qd + off, kd + off, IDESC_QK, 1u);
    }
  };
  // P·V over keys [32·h, 32·h + 64) of the tile (h = 0: first half, 1: second).
  auto issue_pv_half = [&](int t, int vst, int h, uint32_t acc) {
    // P: 16 keys = 8 TMEM columns (two 16-bit values per column); V: 16 key
    // rows of 128 bytes in each 64-column box, boxes SW128_BOX_BYTES apart.
    const Desc vd = v_desc0 + (Desc)((vst * L::KV_BYTES) >> 4);
    const uint32_t d_o = tmem + TmemO<D>::col(t, 0);
    const uint32_t a_p = tmem + S_COL[t];
    if constexpr (FP8) {
      // P: 32 keys = 8 TMEM columns (four E4M3 values per column); Vᵀ rows
      // hold keys, 32 keys = 32 bytes of each 128-byte row
#pragma unroll
      for (int k = 2 * h; k < 2 * h + 2; ++k)
        mma_ts<true>(d_o, a_p + k * 8, vd + 2 * k, IDESC_PV, k == 0 ? acc : 1u);
      return;
    }
    const int k0 = h * (BN / 32);
    if constexpr (MODE == 0) {  // one asm block (plain kernel)
      umma_ts_lo_x4<SDESC_HI, 8, 128>(d_o, a_p + k0 * 8, vd + k0 * 128, IDESC_PV, acc);
      return;
    }
    mma_ts<false>(d_o, a_p + k0 * 8, vd + ((k0 * 16 * 128) >> 4), IDESC_PV, acc);
#pragma unroll
    for (int k = k0 + 1; k < k0 + BN / 32; ++k)
      mma_ts<false>(d_o, a_p + k * 8, vd + ((k * 16 * 128) >> 4), IDESC_PV, 1u);
  };

  // Phase bits, one per barrier the MMA thread waits on.
  constexpr uint32_t QF = 0, PF = 2, OC = 4, OF = 6, PH = 8;
  uint32_t ph = 0;
  auto wait_flip = [&](int bar, uint32_t bit, uint32_t invert) {
    const bool r = wait_bar_warp(bar_addr(sbase, bar), ((ph >> bit) & 1u) ^ invert, c);
    ph ^= 1u << bit;
    return r;
  };
  Unit U;
  for (int it = 0; ok && next_unit<L::GROUPED>(p, it, U); ++it) {
    const int j0 = U.j0, n0 = U.n[0], n1 = U.n[1], nmax = U.nmax;
    if (nmax == j0) continue;
    const int k0 = st;
    const uint32_t k0_ph = kv_ph;
    if (++st == L::STAGES) { st = 0; kv_ph ^= 1; }
    if (!(ok = wait_bar_warp(bar_addr(sbase, BAR_KV + k0), k0_ph, c))) break;
    if (n0 > j0 && !(ok = wait_flip(BAR_QFULL + 0, QF + 0, 0))) break;
    if (n1 > j0 && !(ok = wait_flip(BAR_QFULL + 2, QF + 1, 0))) break;
    tc_fence_after();
    // Q_t is released (QEMPTY) as soon as the unit's last S_t MMA is issued,
    // so the next unit's Q tile loads while this unit's softmax and P·V run.
    if (n0 > j0) {
      issue_qk(0, k0);
      umma_commit_warp(bar_addr(sbase, BAR_SFULL + 0));
      if (n0 == j0 + 1) umma_commit_warp(bar_addr(sbase, BAR_QEMPTY + 0));
    }
    if (n1 > j0) {
      issue_qk(1, k0);
      umma_commit_warp(bar_addr(sbase, BAR_SFULL + 1));
      if (n1 == j0 + 1) umma_commit_warp(bar_addr(sbase, BAR_QEMPTY + 2));
    }
    umma_commit_warp(bar_addr(sbase, BAR_KV + L::STAGES + k0));

    for (int j = j0; j < nmax && ok; ++j) {
      const int vs = st;
      const uint32_t vs_ph = kv_ph;
      if (++st == L::STAGES) { st = 0; kv_ph ^= 1; }
      int kn = -1;
      uint32_t kn_ph = 0;
      if (j + 1 < nmax) {
        kn = st;
        kn_ph = kv_ph;
        if (++st == L::STAGES) { st = 0; kv_ph ^= 1; }
      }
      if (!(ok = wait_bar_warp(bar_addr(sbase, BAR_KV + vs), vs_ph, c))) break;
      bool kn_ready = false;
      for (int t = 0; t < 2; ++t) {
        const int nt = t ? n1 : n0;
        if (j >= nt) continue;
        if (!(ok = wait_flip(BAR_PHALF + t, PH + t, 0))) break;
        if (j > j0) {
          if constexpr (!L::SELF_RESCALE)
            if (!(ok = wait_flip(BAR_OCORR + t, OC + t, 0))) break;
        } else {
          if (!(ok = wait_flip(BAR_OFREE + 2 * t, OF + t, 1))) break;
        }
        tc_fence_after();
        issue_pv_half(t, vs, 0, j > j0 ? 1u : 0u);
        if (!(ok = wait_flip(BAR_PFULL + t, PF + t, 0))) break;
        tc_fence_after();
        issue_pv_half(t, vs, 1, 1u);
        if (j == nt - 1) {
          umma_commit_warp(bar_addr(sbase, BAR_PVDONE + 2 * t));
        } else {
          if (!kn_ready) {
            if (!(ok = wait_bar_warp(bar_addr(sbase, BAR_KV + kn), kn_ph, c))) break;
            kn_ready = true;
            tc_fence_after();
          }
          issue_qk(t, kn);
          umma_commit_warp(bar_addr(sbase, BAR_SFULL + t));
          if (j + 2 == nt) umma_commit_warp(bar_addr(sbase, BAR_QEMPTY + 2 * t));
        }
      }
      if (!ok) break;
      umma_commit_warp(bar_addr(sbase, BAR_KV + L::STAGES + vs));
      if (kn >= 0) umma_commit_warp(bar_addr(sbase, BAR_KV + L::STAGES + kn));
    }
  }
  if (!ok) {
    // Let every issued MMA finish before TMEM is released.
    volatile int no_abort = 0;
    Ctl drain{&no_abort, 100000000ull};
    umma_commit_warp(bar_addr(sbase, BAR_DRAIN));
    wait_bar_warp(bar_addr(sbase, BAR_DRAIN), 0, drain);
  }
}

// ================================================================= softmax
// Rounds (lo, hi) to the 16-bit MMA type and packs them as one TMEM column
// (lo in the low half).
template <bool BF16>
__device__ __forceinline__ uint32_t round_pack(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

// Row max of one S tile for this thread's row, in log2 units of the scaled
// score. MASKED: keys c >= nvalid are masked, and s is rewritten in place to
// s·scale·log2e (−inf where masked); otherwise s stays raw and the max of the
// scaled row is max(s)·k, valid for k >= 0 (a negative scale always takes
// the masked form, with every key of an interior tile valid).
template <bool MASKED>
__device__ __forceinline__ float row_max(uint32_t (&s)[BN], float sl2, int nvalid) {
  float mx[8];
  if constexpr (!MASKED) {
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(s[i]);
#pragma unroll
    for (int i = 8; i < BN; i += 2)
      mx[(i >> 1) & 7] = fmax3(mx[(i >> 1) & 7], __uint_as_float(s[i]), __uint_as_float(s[i + 1]));
    return fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * sl2;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
    for (int i = 0; i < BN; i += 2) {
      const float v0 = i < nvalid ? __uint_as_float(s[i]) * sl2 : -INFINITY;
      const float v1 = i + 1 < nvalid ? __uint_as_float(s[i + 1]) * sl2 : -INFINITY;
      s[i] = __float_as_uint(v0);
      s[i + 1] = __float_as_uint(v1);
      mx[(i >> 1) & 7] = fmax3(mx[(i >> 1) & 7], v0, v1);
    }
    return fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
  }
}

// Bias mode: s·scale·log2e + bias·log2e for this thread's row, −inf for keys
// c >= nvalid, written over s; returns the row max (log2 units). brow is the
// row in the bias buffer (first 64-column box); its 16-byte chunks sit at
// chunk ^ (row & 7), the 128-byte swizzle the TMA load applied.
template <bool BF16>
__device__ __forceinline__ float row_max_bias(uint32_t (&s)[BN], float sl2, int nvalid,
                                              const uint8_t* brow, int sw) {
  constexpr float LOG2E = 1.4426950408889634f;
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
  for (int c = 0; c < BN / 8; ++c) {
    const uint4 bv = *reinterpret_cast<const uint4*>(brow + (c >> 3) * SW128_BOX_BYTES +
                                                     (((c & 7) ^ sw) << 4));
    const uint32_t w[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = c * 8 + 2 * e;
      float b0, b1;
      if constexpr (BF16) {
        b0 = __uint_as_float(w[e] << 16);
        b1 = __uint_as_float(w[e] & 0xffff0000u);
      } else {
        b0 = __half2float(__ushort_as_half((unsigned short)(w[e] & 0xffffu)));
        b1 = __half2float(__ushort_as_half((unsigned short)(w[e] >> 16)));
      }
      const float v0 = i < nvalid ? fmaf(__uint_as_float(s[i]), sl2, b0 * LOG2E) : -INFINITY;
      const float v1 = i + 1 < nvalid ? fmaf(__uint_as_float(s[i + 1]), sl2, b1 * LOG2E) : -INFINITY;
      s[i] = __float_as_uint(v0);
      s[i + 1] = __float_as_uint(v1);
      mx[(i >> 1) & 7] = fmax3(mx[(i >> 1) & 7], v0, v1);
    }
  }
  return fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
}

// O ← α·O for this thread's row of O in TMEM (t_o: this warp's lanes), when
// any row of the warp has α ≠ 1. The caller has waited for this step's S, so
// the previous P·V into O is complete; its arrival on the half-P barrier,
// which follows, lets the next P·V start.
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t t_o, float alpha) {
  if (!__any_sync(0xffffffffu, alpha != 1.f)) return;
#pragma unroll 1
  for (int q = 0; q < D / 16; ++q) {  // 16 columns at a time: S is still half in registers
    uint32_t o[16];
    tmem_ld_x16(t_o + 16 * q, o);
    tmem_wait_ld();
    reg_pin_x16(o);
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
    tmem_st_x16(t_o + 16 * q, o);
  }
}

// P = exp2(s·scale·log2e − mref) for this thread's row, rounded to 16 bits and
// written over S in TMEM in two 64-key halves (arriving on half_bar after the
// first, and after rescaling O by alpha); returns the sum of the unrounded P.
// Scale-and-subtract and the sum use packed fp32 pairs.
template <int D, bool BF16, bool MASKED, bool RESCALE>
__device__ __forceinline__ float exp_store(const uint32_t (&s)[BN], float sl2, float mref,
                                           uint32_t t_p, uint32_t half_bar, uint32_t t_o,
                                           float alpha) {
  const uint64_t k2 = f2_pack(sl2, sl2), nm2 = f2_pack(-mref, -mref);
  uint64_t acc[4] = {0, 0, 0, 0};
  uint32_t pk[BN / 2];
#pragma unroll
  for (int i = 0; i < BN / 2; ++i) {
    const uint64_t x = ((uint64_t)s[2 * i + 1] << 32) | s[2 * i];
    const uint64_t y = MASKED ? fadd2(x, nm2) : ffma2(x, k2, nm2);
    const float p0 = ex2_approx(f2_lo(y)), p1 = ex2_approx(f2_hi(y));
    acc[i & 3] = fadd2(acc[i & 3], f2_pack(p0, p1));
    pk[i] = round_pack<BF16>(p0, p1);
    if (i == BN / 4 - 1) {
      // First 64 keys: store and signal now, so the P·V MMA on them can
      // overlap the second half of the exponentials.
      tmem_st_x32(t_p, pk);
      if constexpr (RESCALE) rescale_o<D>(t_o, alpha);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(half_bar);
    }
    if (i == 3 * BN / 8 - 1) tmem_st_x16(t_p + 32, pk + 32);
  }
  tmem_st_x16(t_p + 48, pk + 48);
  const uint64_t e2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
  return f2_lo(e2) + f2_hi(e2);
}

// FP8 form of exp_store: P rounded to E4M3 (four keys per TMEM column, 32
// columns per tile), first 64 keys stored and signalled early. Returns the sum
// of the unrounded P (LSE) and, in *qsum, the sum of the rounded P — the exact
// denominator of the P·V product the tensor core forms from them.
template <int D, bool MASKED>
__device__ __forceinline__ float exp_store_f8(const uint32_t (&s)[BN], float sl2, float mref,
                                              uint32_t t_p, uint32_t half_bar, float* qsum,
                                              uint32_t t_o, float alpha) {
  const uint64_t k2 = f2_pack(sl2, sl2), nm2 = f2_pack(-mref, -mref);
  uint64_t acc[2] = {0, 0}, accq[2] = {0, 0};
  uint32_t pk[BN / 4];
#pragma unroll
  for (int w = 0; w < BN / 4; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 2 * w + h;
      const uint64_t x = ((uint64_t)s[2 * i + 1] << 32) | s[2 * i];
      const uint64_t y = MASKED ? fadd2(x, nm2) : ffma2(x, k2, nm2);
      const float p0 = ex2_approx(f2_lo(y)), p1 = ex2_approx(f2_hi(y));
      acc[h] = fadd2(acc[h], f2_pack(p0, p1));
      const uint32_t q = e4m3x2(p0, p1);
      accq[h] = fadd2(accq[h], e4m3x2_to_f2(q));
      word |= q << (16 * h);
    }
    pk[w] = word;
    if (w == BN / 8 - 1) {
      tmem_st_x16(t_p, pk);
      rescale_o<D>(t_o, alpha);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(half_bar);
    }
  }
  tmem_st_x16(t_p + 16, pk + 16);
  const uint64_t q2 = fadd2(accq[0], accq[1]);
  *qsum = f2_lo(q2) + f2_hi(q2);
  const uint64_t e2 = fadd2(acc[0], acc[1]);
  return f2_lo(e2) + f2_hi(e2);
}

// x rounded to the 16-bit MMA type and back.
template <bool BF16>
__device__ __forceinline__ float round16(float x) {
  if constexpr (BF16) return __bfloat162float(__float2bfloat16_rn(x));
  else return __half2float(__float2half_rn(x));
}

template <int D, bool BF16, int MODE>
__device__ void role_softmax(const Params& p, uint8_t* smem, uint32_t sbase, uint32_t tmem,
                             const Ctl& c, int t) {
  using L = Layout<D, MODE>;
  constexpr bool BIAS = L::BIAS, FP8 = L::FP8;
  (void)BIAS;
  (void)FP8;
  const int r = threadIdx.x & 127;                           // row within the Q tile
  const uint32_t lane_base = (uint32_t)((threadIdx.x >> 5) & 3) * 32;
  const uint32_t t_s = tmem + (lane_base << 16) + S_COL[t];  // this warp's lanes of S_t / P_t
  float4* stats = reinterpret_cast<float4*>(smem + L::OFF_STATS);
  float* alpha_s = reinterpret_cast<float*>(smem + L::OFF_ALPHA) + t * BM;
  (void)alpha_s;
  const float sl2 = p.scale_log2;
  uint32_t sf_ph = 0, bf_ph = 0;
  int units_done = 0;
  const uint8_t* brow = smem + L::OFF_BIAS + t * L::BIAS_BYTES + r * 128;
  Unit U;
  for (int it = 0; get_unit_warp<L::RING, L::GROUPED>(p, smem, sbase, it, c, U) > 0; ++it) {
    if (!tile_active(U, t)) continue;
    const int row = U.mb[t] * BM + r;
    // this warp's lanes of the unit's O buffer (the k-th unit of the tile uses buffer k mod BUFS)
    const uint32_t t_o =
        tmem + (lane_base << 16) + TmemO<D>::col(t, units_done & (TmemO<D>::BUFS - 1));
    // l_e: sum of the unrounded P (gives LSE). l_o normalises O: l_e plus,
    // per K/V tile, the rounding error of that tile's largest P (the weight
    // that dominates a peaked row), so that O divides the P·V sum by a
    // denominator built from the same 16-bit weights where it matters.
    float m = -INFINITY, l_o = 0.f, l_e = 0.f;
    for (int j = U.j0; j < U.n[t]; ++j) {
      if (!wait_bar_warp(bar_addr(sbase, BAR_SFULL + t), sf_ph, c)) return;
      sf_ph ^= 1;
      tc_fence_after();
      uint32_t s[BN];
#pragma unroll
      for (int q = 0; q < BN / 32; ++q) tmem_ld_x32(t_s + 32 * q, s + 32 * q);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < BN / 32; ++q) reg_pin_x32(s + 32 * q);

      bool masked;
      float m_cand;
      if constexpr (BIAS) {
        // Every tile adds its bias block, so every tile takes the masked form.
        masked = true;
        int limit = U.key_len;
        if (p.s.causal) limit = min(limit, row + 1);
        if (!wait_bar_warp(bar_addr(sbase, BAR_BFULL + t), bf_ph, c)) return;
        bf_ph ^= 1;
        m_cand = row_max_bias<BF16>(s, sl2, limit - j * BN, brow, r & 7);
        mbar_arrive(bar_addr(sbase, BAR_BEMPTY + t));
      } else {
        masked = sl2 < 0.f || tile_needs_mask(p.s, U, t, j);
        int nvalid = 0;
        if (masked) {
          int limit = U.key_len;
          if (p.s.causal) limit = min(limit, row + 1);
          nvalid = limit - j * BN;  // keys c < nvalid of this tile are allowed
        }
        m_cand = masked ? row_max<true>(s, sl2, nvalid) : row_max<false>(s, sl2, 0);
      }
      // Keep the old reference max unless the new one is RESCALE_THRESHOLD
      // (log2) above it: O and l share the reference, so the result is
      // unchanged, P stays below 2^8 and the O rescale is skipped.
      const float m_new = (m_cand > m + RESCALE_THRESHOLD) ? m_cand : m;
      // α rescales O before the P·V of this tile may start (in exp_store, or
      // by the correction warps); the first tile of a unit starts O afresh
      float alpha = 1.f;
      if constexpr (L::SELF_RESCALE) {
        if (m_new != m && j > U.j0) alpha = ex2_approx(m - m_new);
      } else {
        if (m_new != m) alpha = ex2_approx(m - m_new);
        if (j > U.j0) {
          alpha_s[r] = alpha;
          mbar_arrive(bar_addr(sbase, BAR_AFULL + t));
        }
      }
      m = m_new;
      const float mref = (m == -INFINITY) ? 0.f : m;
      const uint32_t half_bar = bar_addr(sbase, BAR_PHALF + t);
      if constexpr (FP8) {
        float qsum;
        const float lsum =
            masked ? exp_store_f8<D, true>(s, sl2, mref, t_s, half_bar, &qsum, t_o, alpha)
                   : exp_store_f8<D, false>(s, sl2, mref, t_s, half_bar, &qsum, t_o, alpha);
        tmem_wait_st();
        l_e = l_e * alpha + lsum;
        l_o = l_o * alpha + qsum;
      } else {
        constexpr bool RS = L::SELF_RESCALE;
        const float lsum = masked ? exp_store<D, BF16, true, RS>(s, sl2, mref, t_s, half_bar, t_o, alpha)
                                  : exp_store<D, BF16, false, RS>(s, sl2, mref, t_s, half_bar, t_o, alpha);
        const float pmax = ex2_approx(m_cand - mref);  // this tile's largest P
        const float delta = round16<BF16>(pmax) - pmax;
        tmem_wait_st();
        l_e = l_e * alpha + lsum;
        l_o = l_o * alpha + (lsum + delta);
      }
      tc_fence_before();
      mbar_arrive(bar_addr(sbase, BAR_PFULL + t));
    }
    // One barrier per stats buffer. The first S of unit k is issued after the
    // first P·V of unit k - 1, which waited for the epilogue of unit
    // k - 1 - BUFS to free its O buffer (that epilogue read its stats first);
    // with NSTATS >= BUFS + 1 buffers, buffer k mod NSTATS is rewritten only
    // after its previous contents were read, so no barrier runs a phase ahead.
    constexpr int NSTATS = TmemO<D>::NSTATS;
    const int buf = units_done & (NSTATS - 1);
    stats[(buf * 2 + t) * BM + r] = make_float4(m, l_o, l_e, 0.f);
    ++units_done;
    mbar_arrive(bar_addr(sbase, BAR_STATS + 4 * t + buf));
  }
}

// ====================================================== correction/epilogue
template <int D, bool BF16>
__device__ __forceinline__ uint32_t cvt2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

template <int D, bool BF16, int MODE>
__device__ void role_correction(const Params& p, uint8_t* smem, uint32_t sbase, uint32_t tmem,
                                const Ctl& c, const CUtensorMap* tm_o) {
  using L = Layout<D, MODE>;
  constexpr bool BIAS = L::BIAS, FP8 = L::FP8;
  (void)BIAS;
  (void)FP8;
  const int r = threadIdx.x & 127;
  const int wl = (threadIdx.x >> 5) & 3;  // warp within the group = 32-row slab
  const int lane = threadIdx.x & 31;
  const uint32_t lane_base = (uint32_t)wl * 32;
  const float4* stats = reinterpret_cast<const float4*>(smem + L::OFF_STATS);
  constexpr int OBUF = TmemO<D>::BUFS, NSTATS = TmemO<D>::NSTATS;
  const float* alpha_all = reinterpret_cast<const float*>(smem + L::OFF_ALPHA);
  uint32_t af_ph[2] = {0, 0}, pv_ph = 0;  // pv_ph: one bit per (tile, O buffer)
  (void)alpha_all;
  (void)af_ph;
  int units_done[2] = {0, 0};
  int ost = 0;  // staging buffer toggle (per warp)
  bool ok = true;
  Unit U;
  for (int it = 0; ok; ++it) {
    const int got = get_unit_warp<L::RING, L::GROUPED>(p, smem, sbase, it, c, U);
    if (got <= 0) {
      ok = got == 0;
      break;
    }
    // O buffer of each tile for this unit (units with the tile active, mod OBUF)
    const int obuf[2] = {units_done[0] & (OBUF - 1), units_done[1] & (OBUF - 1)};
    // ---- rescale O_t for every K/V tile after the first (when the softmax does not)
    if constexpr (!L::SELF_RESCALE) {
      for (int j = U.j0 + 1; j < U.nmax && ok; ++j) {
        for (int t = 0; t < 2; ++t) {
          if (j >= U.n[t]) continue;
          if (!(ok = wait_bar_warp(bar_addr(sbase, BAR_AFULL + t), af_ph[t], c))) break;
          af_ph[t] ^= 1;
          const float a = alpha_all[t * BM + r];
          if (__any_sync(0xffffffffu, a != 1.f)) {
            tc_fence_after();
            const uint32_t t_o = tmem + (lane_base << 16) + TmemO<D>::col(t, obuf[t]);
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
              uint32_t o[32];
              tmem_ld_x32(t_o + 32 * q, o);
              tmem_wait_ld();
              reg_pin_x32(o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * a);
              tmem_st_x32(t_o + 32 * q, o);
            }
            tmem_wait_st();
          }
          tc_fence_before();
          mbar_arrive(bar_addr(sbase, BAR_OCORR + t));
        }
      }
      if (!ok) break;
    }
    // ---- epilogue: O / l -> 16-bit -> smem (64-byte swizzle) -> TMA store; LSE
    for (int t = 0; t < 2 && ok; ++t) {
      if (!U.present[t]) continue;
      const int row = U.mb[t] * BM + r;
      const int head = U.b * p.s.Hq + U.hq[t];
      float inv_l = 0.f, lse = -INFINITY;
      const bool has = tile_active(U, t);
      const int ob = obuf[t];
      if (has) {
        const int k = units_done[t]++, buf = k & (NSTATS - 1);
        if (!(ok = wait_bar_warp(bar_addr(sbase, BAR_STATS + 4 * t + buf), (k / NSTATS) & 1, c)))
          break;
        const float4 ml = stats[(buf * 2 + t) * BM + r];
        const int pb = 2 * t + ob;
        if (!(ok = wait_bar_warp(bar_addr(sbase, BAR_PVDONE + pb), (pv_ph >> pb) & 1, c))) break;
        pv_ph ^= 1u << pb;
        tc_fence_after();
        if (ml.y > 0.f) {
          inv_l = __frcp_rn(ml.y);
          if constexpr (FP8) inv_l *= p.o_scale;
          lse = (ml.x + __log2f(ml.z)) * 0.69314718055994531f;
        }
      }
      const int slab_row0 = U.mb[t] * BM + 32 * wl;
      const uint32_t t_o = tmem + (lane_base << 16) + TmemO<D>::col(t, ob);
      if (p.o_part != nullptr) {
        // Split-KV: this split's O (normalised by its own l) and LSE, fp32,
        // for the merge kernel; each thread writes its row's 128-byte chunks.
        const size_t prow = ((size_t)U.split * p.s.B * p.s.Hq + head) * p.s.N + row;
#pragma unroll 1
        for (int q = 0; q < D / 32; ++q) {
          uint32_t o[32];
          if (has) {
            tmem_ld_x32(t_o + 32 * q, o);
            tmem_wait_ld();
            reg_pin_x32(o);
            if (q == D / 32 - 1) {
              tc_fence_before();
              mbar_arrive(bar_addr(sbase, BAR_OFREE + 2 * t + ob));
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0u;
          }
          if (row < p.s.N) {
            float4* dst = reinterpret_cast<float4*>(p.o_part + prow * D + 32 * q);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                   __uint_as_float(o[4 * i + 2]) * inv_l, __uint_as_float(o[4 * i + 3]) * inv_l);
          }
        }
        if (row < p.s.N) p.lse_part[prow] = lse;
        continue;
      }
#pragma unroll 1
      for (int q = 0; q < D / 32; ++q) {
        uint32_t o[32];
        if (has) {
          tmem_ld_x32(t_o + 32 * q, o);
          tmem_wait_ld();
          reg_pin_x32(o);
          if (q == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar_addr(sbase, BAR_OFREE + 2 * t + ob));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = cvt2<D, BF16>(__uint_as_float(o[2 * i]) * inv_l,
                                __uint_as_float(o[2 * i + 1]) * inv_l);
        uint8_t* buf = smem + L::OFF_OST + (wl * 2 + ost) * OST_BYTES;
        if (lane == 0) bulk_wait_group_read<1>();  // the store that used `buf` last has read it
        __syncwarp();
        // row `lane`, 16-byte chunk k lands at chunk k ^ ((row >> 1) & 3): 64-byte swizzle
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint4 v = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          *reinterpret_cast<uint4*>(buf + lane * 64 + ((k ^ ((lane >> 1) & 3)) * 16)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && slab_row0 < p.s.N) {
          tma_store_3d(tm_o, smem_addr(buf), 32 * q, slab_row0, head);
          bulk_commit_group();
        }
        ost ^= 1;
      }
      if (p.lse != nullptr && row < p.s.N) p.lse[(size_t)head * p.s.N + row] = lse;
    }
  }
  if (lane == 0) bulk_wait_group<0>();
  __syncwarp();
}

// ================================================================== kernel
template <int D, bool BF16, int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const __grid_constant__ CUtensorMap tm_b, const Params p) {
  using L = Layout<D, MODE>;
  constexpr bool BIAS = L::BIAS, FP8 = L::FP8;
  (void)BIAS;
  (void)FP8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(bar_addr(sbase, BAR_QFULL + 2 * t + b), 1);
        mbar_init(bar_addr(sbase, BAR_QEMPTY + 2 * t + b), 1);
      }
      mbar_init(bar_addr(sbase, BAR_SFULL + t), 1);
      mbar_init(bar_addr(sbase, BAR_PFULL + t), BM);
      mbar_init(bar_addr(sbase, BAR_PHALF + t), BM);
      mbar_init(bar_addr(sbase, BAR_AFULL + t), BM);
      mbar_init(bar_addr(sbase, BAR_OCORR + t), BM);
      for (int b = 0; b < 2; ++b) {
        mbar_init(bar_addr(sbase, BAR_PVDONE + 2 * t + b), 1);
        mbar_init(bar_addr(sbase, BAR_OFREE + 2 * t + b), BM);
      }
      for (int b = 0; b < 4; ++b) mbar_init(bar_addr(sbase, BAR_STATS + 4 * t + b), BM);
      mbar_init(bar_addr(sbase, BAR_BFULL + t), 1);
      mbar_init(bar_addr(sbase, BAR_BEMPTY + t), BM);
    }
    mbar_init(bar_addr(sbase, BAR_DRAIN), 1);
    // unit records: one writer; one arrival per reading warp (MMA 1, softmax
    // 8, correction 4, and the two bias loaders in bias mode)
    for (int u = 0; u < UNIT_RING; ++u) {
      mbar_init(bar_addr(sbase, BAR_UFULL + u), 1);
      mbar_init(bar_addr(sbase, BAR_UEMPTY + u), BIAS ? 15 : 13);
    }
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(bar_addr(sbase, BAR_KV + s), 1);
      mbar_init(bar_addr(sbase, BAR_KV + L::STAGES + s), 1);
    }
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
    tma_prefetch_map(&tm_o);
    if (BIAS) tma_prefetch_map(&tm_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Ctl ctl{abort_flag, p.timeout_ns};

  // Register split: 2×176 (softmax) + 80 (correction) + 80 (MMA, loads) = 4 × 128.
  if (warp < 8) {
    setmaxnreg_inc<176>();
    role_softmax<D, BF16, MODE>(p, smem, sbase, tmem, ctl, warp >> 2);
  } else if (warp < 12) {
    setmaxnreg_dec<80>();
    role_correction<D, BF16, MODE>(p, smem, sbase, tmem, ctl, &tm_o);
  } else {
    setmaxnreg_dec<80>();
    if (warp == 12) role_mma<D, BF16, MODE>(p, smem, sbase, tmem, ctl);
    if (warp == 13 && lane == 0) role_load<D, MODE>(p, smem, sbase, ctl, &tm_q, &tm_k, &tm_v);
    if constexpr (BIAS) {
      if (warp >= 14 && lane == 0) role_bias_load<D>(p, smem, sbase, ctl, &tm_b, warp - 14);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Bounded-wait self test: one thread waits on a barrier nothing arrives at.
__global__ void fa_wait_selftest_kernel(unsigned long long timeout_ns, int* out) {
  __shared__ alignas(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_addr(&bar), 1);
    mbar_init_fence();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    Ctl c{&abort_flag, timeout_ns};
    const bool ok = wait_bar(smem_addr(&bar), 0, c);
    out[0] = ok ? 1 : 0;
    out[1] = abort_flag;
  }
}

// Split-KV merge: for each query row, combines the splits' partial results
// (O_s normalised by its own denominator, LSE_s natural log; LSE_s = −inf for
// a split with no allowed key) into O = Σ_s e^{LSE_s − m} O_s / Σ_s e^{LSE_s − m}
// and LSE = m + ln Σ_s e^{LSE_s − m}, m = max_s LSE_s — one more step of the
// online recurrence with a whole split as the tile. One warp per row, each
// lane D/32 consecutive elements.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) fa_merge_splits_kernel(const float* __restrict__ o_part,
                                                              const float* __restrict__ lse_part,
                                                              int splits, long long rows, void* o,
                                                              float* lse) {
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < rows;
       row += nwarps) {
    float m = -INFINITY;
    for (int s = 0; s < splits; ++s) m = fmaxf(m, __ldg(lse_part + s * rows + row));
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    float l = 0.f;
    if (m != -INFINITY) {
      for (int s = 0; s < splits; ++s) {
        const float ls = __ldg(lse_part + s * rows + row);
        if (ls == -INFINITY) continue;
        const float w = expf(ls - m);
        l += w;
        const float* src = o_part + ((long long)s * rows + row) * D + lane * E;
        if constexpr (E == 4) {
          const float4 x = __ldg(reinterpret_cast<const float4*>(src));
          acc[0] += w * x.x; acc[1] += w * x.y; acc[2] += w * x.z; acc[3] += w * x.w;
        } else {
          const float2 x = __ldg(reinterpret_cast<const float2*>(src));
          acc[0] += w * x.x; acc[1] += w * x.y;
        }
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    uint32_t packed[E / 2];
#pragma unroll
    for (int e = 0; e < E / 2; ++e) packed[e] = cvt2<D, BF16>(acc[2 * e] * inv, acc[2 * e + 1] * inv);
    uint16_t* dst = reinterpret_cast<uint16_t*>(o) + row * D + lane * E;
    if constexpr (E == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    else *reinterpret_cast<uint32_t*>(dst) = packed[0];
    if (lse != nullptr && lane == 0) lse[row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

// FP8 mode: V [BH][N][D] bytes -> Vᵀ [BH][D][N], so that the P·V product can
// take V as a K-major operand. 64×64-byte tiles through shared memory.
__global__ void __launch_bounds__(256) fa_transpose_u8_kernel(const uint8_t* __restrict__ v,
                                                              uint8_t* __restrict__ vt, int N, int Dm) {
  __shared__ uint8_t tile[64][65];
  const long long bh = blockIdx.z;
  const int n0 = blockIdx.x * 64, d0 = blockIdx.y * 64;
  const uint8_t* src = v + bh * (long long)N * Dm;
  uint8_t* dst = vt + bh * (long long)N * Dm;
  for (int i = threadIdx.x; i < 64 * 64; i += blockDim.x) {
    const int r = i / 64, cidx = i % 64;  // r: key, cidx: d
    if (n0 + r < N) tile[r][cidx] = src[(long long)(n0 + r) * Dm + d0 + cidx];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 64 * 64; i += blockDim.x) {
    const int r = i / 64, cidx = i % 64;  // r: d, cidx: key
    if (n0 + cidx < N) dst[(long long)(d0 + r) * N + n0 + cidx] = tile[cidx][r];
  }
}

#include "fa_bwd_sm100.cuh"

}  // namespace fa

// The host side (argument checks, tensor maps, launches, the C ABI).
#include "fa_host.cuh"
