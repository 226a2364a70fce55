// Split decode over the packed cache on the tcgen05 tensor cores, with both
// MMA A-operands (key codes, value codes) built in tensor memory.
//
// Work split ("stream-K"): every (sequence b, kv head h) unit contributes
// ceil(len_b / 128) tiles of 128 tokens; the tiles of all units, in (b, h)
// order, are cut into 148 equal contiguous ranges, one per persistent CTA
// (one CTA per SM).  A CTA's range covers one or more unit segments; each
// segment leaves one partial (running max, sum, accumulator per query head)
// in slot (unit + CTA), unique because consecutive units' CTA ranges only
// touch at their ends.  The combine pass merges a unit's slots into one
// softmax over the whole sequence (Dual-QK summary Sec. 3.4).
//
// A tcgen05.mma costs about the same whatever its N (up to 256), so the
// schedule minimises MMA instructions per tile and keeps dependent ones apart:
//   scores: 4 MMAs of kind::i8 (K = 32 = one quantization group each): key
//           codes as u8 in tensor memory x the rotated query as two exact s8
//           pieces (q = delta * (128 q1 + q2)), one s32 accumulator per group,
//           so the per-token group scale applies exactly afterwards;
//   PV:     8 MMAs of kind::f16 (K = 16 tokens each): value codes centred as
//           c - L/2 (exact f16) in tensor memory x P' = p * value scale, spread
//           over independent partial accumulators that stay in tensor memory
//           for a whole segment (one accumulator set per segment parity); the
//           zero point, with the L/2 steps folded in, is summed in registers.
//
// Roles inside a CTA, pipelined over tiles with mbarriers:
//   producer warp   : 1-D bulk async copies of a tile's kept key-code rows
//                     (Dual-QK Sec. 3.3: channel-major rows, read selectively),
//                     value-code rows, key and value scale/zero pairs and
//                     channel 0 into one stage of a deep shared-memory ring;
//   key warps (4)   : thread = token: the token's key codes -> u8 -> tensor
//                     memory (lane = token); at a segment start also the
//                     query operand (dropped channel groups zeroed), its
//                     per-head step and its per-group sums;
//   value warps (4) : thread = channel: the channel's 128 value codes -> f16
//                     -> tensor memory (lane = channel);
//   UMMA warp       : the score MMAs one tile ahead, then the PV MMAs;
//   epilogue warps  : thread = (token, heads): score = delta * sum_g s_g S_g +
//                     sum_g z_g sum(q_g) (+ q_0 k_0), online softmax with a
//                     lazily raised max, P' into shared memory, the value
//                     zero-point terms sum_t p_t z_t in registers; when the max
//                     rises inside a segment, thread = (channel, heads) rescales
//                     the segment's PV accumulator in tensor memory; two tiles
//                     after a segment ends, the accumulator is read out into
//                     the segment's partial.
// Scores come straight from the codes; no dequantized key is ever formed
// (tq-kv abstract; Dual-QK summary Sec. 3.2, 3.3).  Every mbarrier wait is
// bounded; after a give-up all waits fall through and the CTA writes NaN
// partials instead of hanging.
#include "common.cuh"
#include "sm100.cuh"

namespace kvq {
namespace {

using namespace sm100;

constexpr int kCtas = 148;  // one persistent CTA per SM
constexpr int kTile = 128;
constexpr float kLazyMax = 8.0f;  // the running max is raised only when a score exceeds it by 2^8
constexpr int kMaxStages = 12;
constexpr int kSmemLimit = 227 * 1024;
constexpr float kQSteps = 16000.0f;  // |q| / delta <= 16000: pieces q1 in [-125, 125], q2 in [-64, 63]

template <int G, int KB, int VB, bool CH0>
struct Shape {
  static constexpr int TPT = G > 4 ? 2 : 1;  // epilogue threads per token (head parts)
  static constexpr int HH = G / TPT;         // heads per epilogue thread: 1, 2, 4 or 8
  static constexpr int NGRP = 1;  // epilogue groups, group g taking tiles t with t % NGRP == g (2 measured no faster)
  static constexpr int EPI_WARPS = 4 * TPT * NGRP;
  static constexpr int EPI_THREADS = 32 * EPI_WARPS;
  static constexpr int MMA_WARP = 8 + EPI_WARPS;
  static constexpr int PROD_WARP = MMA_WARP + 1;
  static constexpr int THREADS = 32 * (PROD_WARP + 1);
  static constexpr int NS = 2 * G < 16 ? 16 : 2 * G;  // score columns per group: q1 rows, then q2 rows
  static constexpr int NO = 4 * G < 16 ? 16 : 4 * G;  // PV columns: (value group, head)
  static constexpr int KST = G > 8 ? 1 : 2;  // key operand stages in tensor memory
  static constexpr int VST = G > 8 ? 1 : 2;  // value operand stages in tensor memory
  static constexpr int SB = 2;               // score accumulator buffers
  static constexpr int LA = SB - 1;          // score MMAs are issued LA tiles ahead of the PV MMAs
  static constexpr int NKR = KST > 1 ? KST : 2;  // key-ready barriers
  static constexpr int OB = 2;                        // PV accumulator sets: one per segment parity
  static constexpr int PP = G > 8 ? 1 : 2;  // partial accumulators per PV (independent chains)
  // tensor-memory columns; every accumulator starts at a multiple of its width
  static constexpr int TM_AK = 0;                                  // KST key stages x 32 columns (128 u8 codes)
  static constexpr int TM_AV = 32 * KST;                           // VST value stages x 64 columns (128 f16 codes)
  static constexpr int TM_S = (TM_AV + 64 * VST + 63) / 64 * 64;   // SB score buffers x 4 groups x NS
  static constexpr int TM_O = TM_S + SB * 4 * NS;                  // NGRP x 2 PV sets x PP partials x NO
  static constexpr int TMEM_COLS = 512;
  static_assert(TM_AK + 32 * KST <= TM_AV && TM_AV + 64 * VST <= TM_S, "operand columns");
  static_assert(SB >= LA + 1 && KST >= 1 && VST <= 2, "stage counts");
  static_assert(TM_O + NGRP * OB * PP * NO <= TMEM_COLS, "tensor memory");
  static_assert(TM_S % NS == 0 && TM_O % NO == 0, "accumulator alignment");
  // one ring stage: key-code rows, value-code rows, key (scale, zero) rows,
  // value (scale, zero) per token, channel 0
  static constexpr int KROW = kTile * (KB == 4 ? 2 : 1);  // bytes of one key row (4 channels)
  static constexpr int VROW = kTile * VB / 8;             // bytes of one value row (1 channel)
  static constexpr int R_KC = 0;
  static constexpr int R_VC = R_KC + kPruneGroups * KROW;
  static constexpr int R_KS = R_VC + kHeadDim * VROW;
  static constexpr int R_VS = R_KS + kGroups * kTile * 4;
  static constexpr int R_K0 = R_VS + kTile * kGroups * 4;
  static constexpr int STAGE = (R_K0 + (CH0 ? kTile * 2 : 0) + 127) / 128 * 128;
  // fixed region behind the ring
  static constexpr int BQ_BYTES = NS * kHeadDim;     // s8 query operand: NS rows x 128 channels
  static constexpr int BP_BYTES = NO * kTile * 2;    // one f16 P' operand
  // query data per segment, double-buffered by segment parity
  static constexpr int QV = (G * 4 + 15) / 16 * 16;  // bytes of G floats, rounded to 16
  static constexpr int F_BQ = 0;                     // [2] query operands
  static constexpr int F_BP = F_BQ + 2 * BQ_BYTES;   // [2] P' buffers
  static constexpr int F_QS = F_BP + 2 * BP_BYTES;   // [2][G][4] f32: per-group sums of the kept q
  static constexpr int F_Q0 = F_QS + 2 * G * 16;     // [2][G] f32: q_0 (channel 0 kept in bf16)
  static constexpr int F_QD = F_Q0 + 2 * QV;         // [2][G] f32: delta of the query pieces
  static constexpr int F_RED = F_QD + 2 * QV;        // [2 tiles][TPT][4 warps][16] f32
  static constexpr int F_RED2 = F_RED + 2 * TPT * 4 * 16 * 4;         // [NGRP][TPT][4 warps][16] f32
  static constexpr int F_PEND = F_RED2 + NGRP * TPT * 4 * 16 * 4;     // [NGRP][2 segment parities][TPT][6 HH] f32
  static constexpr int F_BAR = (F_PEND + NGRP * 2 * TPT * 6 * HH * 4 + 15) / 16 * 16;
  // kready[3] vready[2] pready[2] sdone[3] pvdone[2] qready[2] qfree[2]
  static constexpr int NBAR_FIXED = 16;
  static constexpr int F_REST_NO_RING = F_BAR + NBAR_FIXED * 8 + 16;  // + tmem slot, error flag
  static constexpr int STAGES_FIT = (kSmemLimit - F_REST_NO_RING - 2 * kMaxStages * 8) / STAGE;
  static constexpr int STAGES = STAGES_FIT < kMaxStages ? STAGES_FIT : kMaxStages;
  static_assert(STAGES >= 3, "ring too shallow");
  static constexpr int NBAR = NBAR_FIXED + 2 * STAGES;
  static constexpr int F_SLOT = F_BAR + NBAR * 8;
  static constexpr int F_ERR = F_SLOT + 4;
  static constexpr int FIXED = F_ERR + 12;
  static constexpr int SMEM_BYTES = STAGES * STAGE + FIXED;
  static_assert(SMEM_BYTES <= kSmemLimit, "shared memory");
};

// K position (byte) of channel r of an 8-channel (INT4) or 16-channel (INT2)
// block in the u8 key operand: the 4-bit split puts even channels first, the
// 2-bit split channels r, r+4, r+8, r+12 together.
template <int BITS>
__device__ __forceinline__ int kpos_of(int r) {
  if (BITS == 4) return (r & 1) * 4 + (r >> 1);
  return 4 * (r & 3) + (r >> 2);
}
// K position of code i of an 8-token (INT4) or 16-token (INT2) block in the
// f16 value operand: the f16 conversion pairs code i with code i + 4 (i + 8).
template <int BITS>
__device__ __forceinline__ int vpos_of(int i) {
  if (BITS == 4) return i < 4 ? 2 * i : 2 * (i - 4) + 1;
  return i < 8 ? 2 * i : 2 * (i - 8) + 1;
}
// byte offset of element (row r, byte k) in a K-major 8-bit operand with 128 K bytes
__device__ __forceinline__ uint32_t kmajor8(int r, int k) {
  return (r & 7) * 16 + (k & 15) + (k >> 4) * 128 + (r >> 3) * 1024;
}
// byte offset of element (mn, k) in an MN-major f16 operand with 128 K elements
__device__ __forceinline__ uint32_t mnmajor(int mn, int k) {
  return (mn & 7) * 2 + (k & 7) * 16 + (mn >> 3) * 2048 + (k >> 3) * 128;
}

__device__ __forceinline__ int tiles_of(const DecodeArgs& a, int b) {
  const int len = min(max(a.seq_lens[b], 0), a.max_len);
  return (len + kTile - 1) / kTile;
}

// Walks this CTA's tile range [g, g_end) unit by unit.  Every role keeps its
// own copy and advances it in lock step, so all agree on each tile's unit,
// position and segment flags.
struct TileIter {
  int g, g_end, b, h, i, tiles_b, len;
  uint32_t msk;  // kept channel groups of the current unit
  bool first, last;

  __device__ void load_mask(const DecodeArgs& a) { msk = a.mask ? a.mask[(size_t)b * a.c.H + h] : kFull; }

  __device__ void init(const DecodeArgs& a, int g0, int g1) {
    g = g0;
    g_end = g1;
    if (g >= g_end) return;
    int acc = 0;
    b = 0;
    for (;; ++b) {
      const int t = tiles_of(a, b);
      if (g < acc + a.c.H * t) {
        tiles_b = t;
        break;
      }
      acc += a.c.H * t;
    }
    const int off = g - acc;
    h = off / tiles_b;
    i = off - h * tiles_b;
    len = min(max(a.seq_lens[b], 0), a.max_len);
    load_mask(a);
    first = true;
    last = (i == tiles_b - 1) || (g == g_end - 1);
  }
  __device__ void next(const DecodeArgs& a) {
    ++g;
    if (g >= g_end) return;
    if (++i == tiles_b) {
      i = 0;
      if (++h == a.c.H) {
        h = 0;
        do {
          ++b;
          tiles_b = tiles_of(a, b);
        } while (tiles_b == 0);
        len = min(max(a.seq_lens[b], 0), a.max_len);
      }
    }
    first = (i == 0);
    if (first) load_mask(a);
    last = (i == tiles_b - 1) || (g == g_end - 1);
  }
  __device__ size_t bh(const DecodeArgs& a) const { return (size_t)b * a.c.H + h; }
};

// Bounded wait: tests the phase without blocking first (a completed phase
// costs a few instructions), then waits with try_wait, which suspends the
// thread until the phase completes (or a time hint passes) without taking issue
// slots.  Gives up after about a second, or at once after any earlier give-up
// in the CTA, and reports false.
__device__ __forceinline__ bool ws_wait(uint32_t bar, uint32_t parity, volatile int* err) {
  if (mbar_test_wait(bar, parity)) return true;
#pragma unroll 1
  for (uint32_t it = 0; it < (1u << 21); ++it) {
    if (mbar_try_wait_sleep(bar, parity, 500u)) return true;
    if (*err) return false;
  }
  *err = 1;
  return false;
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
// named barrier that also ORs a predicate over the participating threads
__device__ __forceinline__ bool named_sync_or(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <int G, int KB, int VB, bool CH0, typename In>
__global__ void __launch_bounds__(Shape<G, KB, VB, CH0>::THREADS, 1) k_decode(DecodeArgs a) {
  using S = Shape<G, KB, VB, CH0>;
  constexpr int HH = S::HH, ST = S::STAGES, OB = S::OB, PP = S::PP;
  extern __shared__ __align__(1024) uint8_t smem[];
  const CacheView& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- this CTA's tile range
  int total = 0;
  for (int b = 0; b < c.B; ++b) total += c.H * tiles_of(a, b);
  const int per = (total + kCtas - 1) / kCtas;
  const int g0 = blockIdx.x * per, g1 = min(g0 + per, total);
  if (g0 >= g1) return;
  const int ntiles = g1 - g0;

  uint8_t* fix = smem + ST * S::STAGE;
  const uint32_t bar0 = smem_addr(fix + S::F_BAR);
  // Tile t's barriers: key-ready t % NKR, score-done t % SB, the others t % 2;
  // a wait for tile t takes the parity of t's use of its barrier.
  auto KREADY = [&](int k) { return bar0 + 8 * k; };
  auto VREADY = [&](int k) { return bar0 + 8 * (3 + k); };
  auto PREADY = [&](int k) { return bar0 + 8 * (5 + k); };
  auto SDONE = [&](int k) { return bar0 + 8 * (7 + k); };
  auto PVDONE = [&](int k) { return bar0 + 8 * (10 + k); };  // PV UMMAs of tiles of parity k
  auto QREADY = [&](int k) { return bar0 + 8 * (12 + k); };  // a segment's query data is in buffer k
  auto QFREE = [&](int k) { return bar0 + 8 * (14 + k); };   // the epilogue is done with buffer k
  auto FULL = [&](int s) { return bar0 + 8 * (S::NBAR_FIXED + s); };
  auto EMPTY = [&](int s) { return bar0 + 8 * (S::NBAR_FIXED + ST + s); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fix + S::F_SLOT);
  volatile int* err = reinterpret_cast<volatile int*>(fix + S::F_ERR);

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(FULL(s), 1);
      mbar_init(EMPTY(s), 256 + S::EPI_THREADS / S::NGRP);  // key, value and the tile's epilogue group
    }
    for (int k = 0; k < S::NKR; ++k) mbar_init(KREADY(k), 128);
    for (int k = 0; k < S::SB; ++k) mbar_init(SDONE(k), 1);
    for (int k = 0; k < 2; ++k) {
      mbar_init(VREADY(k), 128);
      mbar_init(PREADY(k), S::EPI_THREADS / S::NGRP);
    }
    for (int k = 0; k < 2; ++k) mbar_init(PVDONE(k), 1);
    for (int k = 0; k < 2; ++k) {
      mbar_init(QREADY(k), 128);
      mbar_init(QFREE(k), S::EPI_THREADS);
    }
    *err = 0;
    mbar_fence_init();
  }
  if (warp == S::MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), S::TMEM_COLS);
    tmem_relinquish();
  }
  // query and P' operands start at zero: their padding rows and columns stay so
  for (int i = tid; i < (2 * S::BQ_BYTES + 2 * S::BP_BYTES) / 16; i += S::THREADS)
    reinterpret_cast<uint4*>(fix + S::F_BQ)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  TileIter it;
  it.init(a, g0, g1);

  if (warp == S::PROD_WARP) {
    // ================================================================ producer
    const int nblk = c.cap / kTile;
    for (int t = 0; t < ntiles; ++t, it.next(a)) {
      const int s = t % ST;
      if (t >= ST) ws_wait(EMPTY(s), ((t / ST) - 1) & 1, err);
      const size_t bh = it.bh(a);
      const uint32_t msk = it.msk;
      const int n0 = it.i * kTile;
      const size_t blk = bh * nblk + it.i;
      const uint32_t dst = smem_addr(smem + s * S::STAGE);
      const bool k0 = CH0 && (msk & 1u);
      if (lane == 0)
        mbar_arrive_expect_tx(FULL(s), (uint32_t)(__popc(msk) * S::KROW + kHeadDim * S::VROW + 2 * kGroups * kTile * 4 +
                                                  (k0 ? kTile * 2 : 0)));
      __syncwarp();
      // one copy per run of adjacent kept channel groups (their rows are adjacent in the block)
      const bool run_start = ((msk >> lane) & 1u) && (lane == 0 || !((msk >> (lane - 1)) & 1u));
      if (run_start) {
        const int run = __ffsll((long long)~((unsigned long long)msk >> lane)) - 1;
        bulk_g2s(dst + S::R_KC + lane * S::KROW, c.kc + key_word_index(bh, c.cap, lane, n0) * (KB == 4 ? 2 : 1),
                 run * S::KROW, FULL(s));
      }
      if (lane == 0) bulk_g2s(dst + S::R_VC, c.vc + blk * kHeadDim * S::VROW, kHeadDim * S::VROW, FULL(s));
      if (lane == 1) bulk_g2s(dst + S::R_KS, c.ks + key_scale_index(bh, c.cap, 0, n0), kGroups * kTile * 4, FULL(s));
      if (lane == 2) bulk_g2s(dst + S::R_VS, c.vs + (bh * c.cap + n0) * kGroups, kTile * kGroups * 4, FULL(s));
      if (k0 && lane == 3) bulk_g2s(dst + S::R_K0, c.k0 + bh * c.cap + n0, kTile * 2, FULL(s));
    }
  } else if (warp == S::MMA_WARP) {
    // ================================================================ UMMA issue
    const uint32_t idesc_s = idesc_u8s8_s32(kTile, S::NS);
    const uint32_t idesc_o = idesc_f16_f32(kTile, S::NO, 0, 1);
    const uint32_t bp = smem_addr(fix + S::F_BP);
    int sseg = -1;    // segment of the tile being scored
    int sstart = 0;   // its first tile
    // bit (t & 3): tile t is its epilogue group's first of the segment / the segment's parity
    uint32_t firstbits = 0, setbits = 0;
    auto score = [&](int t) {
      if (it.first) {
        ++sseg;
        sstart = t;
      }
      firstbits = (firstbits & ~(1u << (t & 3))) | ((t - sstart < S::NGRP ? 1u : 0u) << (t & 3));
      setbits = (setbits & ~(1u << (t & 3))) | ((uint32_t)(sseg & 1) << (t & 3));
      const uint32_t bq = smem_addr(fix + S::F_BQ + (sseg & 1) * S::BQ_BYTES);
      it.next(a);
      ws_wait(KREADY(t % S::NKR), (t / S::NKR) & 1, err);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a0 = tmem + S::TM_AK + (t % S::KST) * 32;
        const uint32_t d0 = tmem + S::TM_S + (t % S::SB) * 4 * S::NS;
        // one MMA per 32-channel group (8 columns of u8 codes, 32 query bytes), all independent
#pragma unroll
        for (int g = 0; g < kGroups; ++g)
          umma_i8_tmem_a(d0 + g * S::NS, a0 + g * 8, smem_desc(bq + g * 256, 128, 1024), idesc_s, 0u);
        umma_commit(SDONE(t % S::SB));
      }
      __syncwarp();
    };
    // The score MMAs of tile t + LA go ahead of the PV MMAs of tile t, so the
    // epilogue finds tile t + 1's scores done while it works on tile t.  Score
    // buffer (t + LA) % SB was last read by the epilogue of tile t + LA - SB
    // <= t - 1, whose P' (PREADY) was waited for in the previous iteration.
    for (int u = 0; u < S::LA && u < ntiles; ++u) score(u);
    for (int t = 0; t < ntiles; ++t) {
      if (t + S::LA < ntiles) score(t + S::LA);
      ws_wait(PREADY(t & 1), (t >> 1) & 1, err);
      ws_wait(VREADY(t & 1), (t >> 1) & 1, err);
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a0 = tmem + S::TM_AV + (t % S::VST) * 64;
        const uint32_t b0 = bp + (t & 1) * S::BP_BYTES;
        // accumulator set: (epilogue group of tile t, segment parity)
        const uint32_t set = (S::NGRP == 2 ? (uint32_t)(t & 1) * OB : 0u) + ((setbits >> (t & 3)) & 1u);
        const uint32_t d0 = tmem + S::TM_O + set * PP * S::NO;
        const bool fresh = (firstbits >> (t & 3)) & 1u;  // the group's first tile of the segment starts its sums
        // 16 tokens per MMA; K step s accumulates into partial s % PP, so
        // consecutive MMAs of one accumulator are PP issues apart
#pragma unroll
        for (int s = 0; s < kTile / 16; ++s)
          umma_f16_tmem_a(d0 + (s % PP) * S::NO, a0 + s * 8, smem_desc(b0 + s * 256, 128, 2048), idesc_o,
                          (fresh && s < PP) ? 0u : 1u);
        umma_commit(PVDONE(t & 1));
      }
      __syncwarp();
    }
  } else if (warp < 4) {
    // ================================================================ key codes -> tensor memory
    const int j = tid;  // token of the tile == tensor-memory lane
    const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
    int kseg = 0;  // segments begun so far
    for (int t = 0; t < ntiles; ++t, it.next(a)) {
      const int s = t % ST;
      const uint8_t* raw = smem + s * S::STAGE + S::R_KC;
      ws_wait(FULL(s), (t / ST) & 1, err);
      // this key stage was read by the score UMMAs of tile t - KST
      if (t >= S::KST) ws_wait(SDONE((t - S::KST) % S::SB), ((t - S::KST) / S::SB) & 1, err);
      tc_fence_after();
      if (it.first) {
        // query data of segment kseg into buffer kseg & 1: per head, delta =
        // max|q| / 16000 and q = delta * (128 q1 + q2) exactly, q1 in row h, q2 in
        // row G + h; dropped channel groups (and channel 0 when it is kept in bf16)
        // are zero.  The buffer was last used by segment kseg - 2, which the
        // epilogue (and so its score UMMAs) finished before freeing it.  Each
        // buffer's two barriers see one phase per use, in order, so no parity wait
        // can pass on a later or an earlier phase.
        const int qb = kseg & 1;
        if (kseg >= 2) ws_wait(QFREE(qb), ((kseg - 2) >> 1) & 1, err);
        uint8_t* BQ = fix + S::F_BQ + qb * S::BQ_BYTES;
        float* qsum = reinterpret_cast<float*>(fix + S::F_QS + qb * G * 16);
        float* q0s = reinterpret_cast<float*>(fix + S::F_Q0 + qb * S::QV);
        float* qds = reinterpret_cast<float*>(fix + S::F_QD + qb * S::QV);
        const uint32_t msk = it.msk;
        for (int hq = warp; hq < G; hq += 4) {
          const In* qrow = static_cast<const In*>(a.q) + ((size_t)it.b * a.Hq + (size_t)it.h * G + hq) * kHeadDim;
          float x[4];
          load_row_warp(qrow, c.rotate != 0, a.inv_sqrt_d, lane, x);
          const bool sel = (msk >> lane) & 1u;
          float v[4], part = 0.0f, amax = 0.0f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            v[i] = sel ? x[i] : 0.0f;
            if (CH0 && lane == 0 && i == 0) v[i] = 0.0f;
            part += v[i];
            amax = fmaxf(amax, fabsf(v[i]));
          }
          amax = warp_max(amax);
          const float delta = amax > 0.0f ? amax / kQSteps : 1.0f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int ch = 4 * lane + i;
            const int qi = __float2int_rn(v[i] / delta);  // |qi| <= 16000
            const int q1 = (qi + 64) >> 7;                // nearest multiple of 128 below qi + 64
            const int q2 = qi - 128 * q1;                 // in [-64, 63]
            constexpr int blk = KB == 4 ? 8 : 16;
            const int p = (ch / blk) * blk + kpos_of<KB>(ch % blk);
            BQ[kmajor8(hq, p)] = (uint8_t)(int8_t)q1;
            BQ[kmajor8(G + hq, p)] = (uint8_t)(int8_t)q2;
          }
#pragma unroll
          for (int m = 1; m < 8; m <<= 1) part += __shfl_xor_sync(kFull, part, m);
          if ((lane & 7) == 0) qsum[hq * kGroups + (lane >> 3)] = part;
          if (lane == 0) {
            q0s[hq] = (CH0 && sel) ? x[0] : 0.0f;
            qds[hq] = delta;
          }
        }
        mbar_arrive(QREADY(qb));  // release: the epilogue reads the data after waiting on it
        ++kseg;
      }
      // every key row is converted: rows of dropped channel groups hold stale
      // codes, which meet zeros in the query operand
      uint32_t r[32];
      if (KB == 4) {
        const uint16_t* kc = reinterpret_cast<const uint16_t*>(raw) + j;
#pragma unroll
        for (int q = 0; q < 16; ++q) {  // channels 8q .. 8q+7: even ones, then odd ones
          const uint32_t x = (uint32_t)kc[(2 * q) * kTile] | ((uint32_t)kc[(2 * q + 1) * kTile] << 16);
          r[2 * q] = x & 0x0F0F0F0Fu;
          r[2 * q + 1] = (x >> 4) & 0x0F0F0F0Fu;
        }
      } else {
        const uint8_t* kc = raw + j;
#pragma unroll
        for (int q = 0; q < 8; ++q) {  // channels 16q .. 16q+15: crumb k of every byte together
          const uint32_t x = (uint32_t)kc[(4 * q) * kTile] | ((uint32_t)kc[(4 * q + 1) * kTile] << 8) |
                             ((uint32_t)kc[(4 * q + 2) * kTile] << 16) | ((uint32_t)kc[(4 * q + 3) * kTile] << 24);
#pragma unroll
          for (int k = 0; k < 4; ++k) r[4 * q + k] = (x >> (2 * k)) & 0x03030303u;
        }
      }
      const uint32_t col = tl + S::TM_AK + (t % S::KST) * 32;
      tmem_st16(col, *reinterpret_cast<const uint32_t(*)[16]>(&r[0]));
      tmem_st16(col + 16, *reinterpret_cast<const uint32_t(*)[16]>(&r[16]));
      tmem_wait_st();
      fence_proxy_async();  // query operand (generic writes) -> tensor core
      tc_fence_before();
      mbar_arrive(KREADY(t % S::NKR));
      mbar_arrive(EMPTY(s));
    }
  } else if (warp < 8) {
    // ================================================================ value codes -> tensor memory
    const int ch = tid - 128;  // channel == tensor-memory lane
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp - 4)) << 16);
    // the 16-byte chunks of a channel's row are stored rotated by channel, so
    // the rows of 8 consecutive channels hit 8 different bank groups
    const int swz = VB == 4 ? (ch >> 1) & 3 : (ch >> 2) & 1;
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % ST;
      const uint8_t* row = smem + s * S::STAGE + S::R_VC + ch * S::VROW;
      ws_wait(FULL(s), (t / ST) & 1, err);
      // this value stage was read by the PV UMMAs of tile t - VST
      if (t >= S::VST) ws_wait(PVDONE((t - S::VST) & 1), ((t - S::VST) >> 1) & 1, err);
      tc_fence_after();
      const uint32_t col = tl + S::TM_AV + (t % S::VST) * 64;
      constexpr int CHUNKS = S::VROW / 16;  // 4 (INT4: 32 tokens each) or 2 (INT2: 64 tokens each)
#pragma unroll
      for (int k = 0; k < CHUNKS; ++k) {
        const uint4 w = *reinterpret_cast<const uint4*>(row + 16 * (k ^ swz));
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
        if (VB == 4) {
          uint32_t rr[16];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t c4[4];
            codes4_to_f16(ws[i], c4);
#pragma unroll
            for (int m = 0; m < 4; ++m) rr[4 * i + m] = c4[m];
          }
          tmem_st16(col + 16 * k, rr);
        } else {
#pragma unroll
          for (int hlf = 0; hlf < 2; ++hlf) {
            uint32_t rr[16];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              uint32_t c8[8];
              codes2_to_f16(ws[2 * hlf + i], c8);
#pragma unroll
              for (int m = 0; m < 8; ++m) rr[8 * i + m] = c8[m];
            }
            tmem_st16(col + 32 * k + 16 * hlf, rr);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(VREADY(t & 1));
      mbar_arrive(EMPTY(s));
    }
  } else if (warp < 8 + S::EPI_WARPS) {
    // ================================================================ epilogue
    // With NGRP epilogue groups, group g takes the tiles t with t % NGRP == g,
    // so one tile's chain of waits and latencies can overlap another's; each
    // group keeps its own online softmax and PV accumulator sets per segment and
    // leaves its own partial, which the combine merges like any other split.
    // (Two groups measured no faster than one at G = 4, so NGRP is 1.)
    const int e = tid - 256;                  // 0 .. EPI_THREADS-1
    const int grp = e / (128 * S::TPT);       // epilogue group
    const int j = e & 127;                    // token (score phase) == tensor-memory lane == channel (PV phase)
    const int part = (e >> 7) % S::TPT;       // head part: heads part*HH .. part*HH + HH - 1
    const int wq = warp & 3;                  // lane quarter == value group in the PV phase
    const int bar_id = 1 + grp * S::TPT + part;
    const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
    // K position of token j in the P' operand (the value conversion's pairing)
    const int pos = VB == 4 ? (j & ~7) + vpos_of<4>(j & 7) : (j & ~15) + vpos_of<2>(j & 15);
    float* red = reinterpret_cast<float*>(fix + S::F_RED);      // [2][TPT][4][16]
    float* red2 = reinterpret_cast<float*>(fix + S::F_RED2) + grp * S::TPT * 64;         // [TPT][4][16]
    float* pend = reinterpret_cast<float*>(fix + S::F_PEND) + grp * 2 * S::TPT * 6 * HH;  // [2][TPT][6 HH]
    const float NEG_INF = -__int_as_float(0x7f800000);

    float m_run[HH], l_acc[HH], zacc[kGroups][HH];
    // this segment's query data for the thread's heads (per-group sums of the
    // kept q, q_0, the step of the query pieces), held in registers when one
    // thread takes a token's heads, else read from shared memory per tile
    constexpr bool QREG = S::TPT == 1;
    float qsg[QREG ? HH : 1][kGroups], q0r[QREG ? HH : 1], qdr[QREG ? HH : 1];
    int nseg = 0;       // segments begun so far
    int qb = 0;         // query buffer and PV accumulator set of the current segment (its parity)
    int seg_tiles = 0;  // tiles of the current segment this group has taken
    int last_own = 0;   // the last tile this group took
    // segments waiting for their read-out: last tile into the set, set, partial slot
    int pn = 0, p0_tile = 0, p0_set = 0, p0_slot = 0, p1_tile = 0, p1_set = 0, p1_slot = 0;
    bool ok = true;
#pragma unroll
    for (int i = 0; i < HH; ++i) {
      m_run[i] = NEG_INF;
      l_acc[i] = 0.0f;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) zacc[g][i] = 0.0f;
    }

    // this thread's PV accumulator columns (channel j, its HH heads) of partial 0 of set os
    auto obase = [&](int os) {
      return tmem + lane_base + S::TM_O + (grp * OB + os) * PP * S::NO + wq * G + part * HH;
    };
    // sum of the PP partials of set os (after the last PV into it completed)
    auto load_out = [&](int os, float (&d)[HH]) {
      const uint32_t base = obase(os);
      if constexpr (PP == 4) {
        uint32_t r[4][HH];
        tmem_ld4_wait<HH>(base, S::NO, r);
#pragma unroll
        for (int i = 0; i < HH; ++i)
          d[i] = (__uint_as_float(r[0][i]) + __uint_as_float(r[1][i])) +
                 (__uint_as_float(r[2][i]) + __uint_as_float(r[3][i]));
      } else if constexpr (PP == 2) {
        uint32_t r0[HH], r1[HH];
        tmem_ld_wait<HH>(base, r0);
        tmem_ld_wait<HH>(base + S::NO, r1);
#pragma unroll
        for (int i = 0; i < HH; ++i) d[i] = __uint_as_float(r0[i]) + __uint_as_float(r1[i]);
      } else {
        uint32_t r0[HH];
        tmem_ld_wait<HH>(base, r0);
#pragma unroll
        for (int i = 0; i < HH; ++i) d[i] = __uint_as_float(r0[i]);
      }
    };
    // a segment that ended at tile tp: its PV output (plus the group's value
    // zero-point term) and its running max and sum into partial slot `slot`
    auto readout = [&](int tp, int os, int slot) {
      ok &= ws_wait(PVDONE(tp & 1), (tp >> 1) & 1, err);
      tc_fence_after();
      float d[HH];
      load_out(os, d);
      tc_fence_before();
      const float nan = __int_as_float(0x7fc00000);
      const bool good = ok && !*err;
      const float* pd = pend + (os * S::TPT + part) * 6 * HH;
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        const size_t row = (size_t)slot * G + part * HH + i;
        a.part_acc[row * kHeadDim + j] = good ? d[i] + pd[(2 + wq) * HH + i] : nan;
        if (j == 0) a.part_ml[row] = good ? make_float2(pd[i], pd[HH + i]) : make_float2(nan, nan);
      }
    };

    // Read out the pending segments whose last PV tile is at least two tiles
    // before tile u.  A set is next written by the group's first tile of the
    // segment after next, at or after u, whose PV follows this tile's P'.
    auto drain = [&](int u) {
      while (pn > 0 && u >= p0_tile + 2) {
        readout(p0_tile, p0_set, p0_slot);
        p0_tile = p1_tile;
        p0_set = p1_set;
        p0_slot = p1_slot;
        --pn;
      }
    };

    for (int t = 0; t < ntiles; ++t, it.next(a)) {
      const int k = t & 1;
      const bool own = S::NGRP == 1 || k == grp;
      if (it.first) {
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          m_run[i] = NEG_INF;
          l_acc[i] = 0.0f;
#pragma unroll
          for (int g = 0; g < kGroups; ++g) zacc[g][i] = 0.0f;
        }
        seg_tiles = 0;
        qb = nseg & 1;  // this segment's query data
        ok &= ws_wait(QREADY(qb), (nseg >> 1) & 1, err);
        ++nseg;
        const float* qsum = reinterpret_cast<const float*>(fix + S::F_QS + qb * G * 16);
        const float* q0s = reinterpret_cast<const float*>(fix + S::F_Q0 + qb * S::QV);
        const float* qds = reinterpret_cast<const float*>(fix + S::F_QD + qb * S::QV);
#pragma unroll
        for (int i = 0; i < (QREG ? HH : 0); ++i) {
          const int hh = part * HH + i;
          const float4 qs = reinterpret_cast<const float4*>(qsum)[hh];
          qsg[i][0] = qs.x;
          qsg[i][1] = qs.y;
          qsg[i][2] = qs.z;
          qsg[i][3] = qs.w;
          q0r[i] = CH0 ? q0s[hh] : 0.0f;
          qdr[i] = qds[hh];
        }
      }
      if (own) {
      drain(t);
      // tokens past the end, and the bf16 window tokens (scored by k_window), take no part
      const int tok = it.i * kTile + j;  // token position in the sequence
      const bool valid = tok < it.len && !in_window(c.sink, c.recent, tok, it.len);
      // per-token scales, zeros and channel 0 from the ring (zero past the sequence end)
      const int s = t % ST;
      ok &= ws_wait(FULL(s), (t / ST) & 1, err);
      const uint8_t* st = smem + s * S::STAGE;
      float2 ksz[kGroups], vsz[kGroups];
#pragma unroll
      for (int g = 0; g < kGroups; ++g)
        ksz[g] = __half22float2(reinterpret_cast<const __half2*>(st + S::R_KS + g * kTile * 4)[j]);
      {
        const uint4 vv = reinterpret_cast<const uint4*>(st + S::R_VS)[j];
        vsz[0] = __half22float2(*reinterpret_cast<const __half2*>(&vv.x));
        vsz[1] = __half22float2(*reinterpret_cast<const __half2*>(&vv.y));
        vsz[2] = __half22float2(*reinterpret_cast<const __half2*>(&vv.z));
        vsz[3] = __half22float2(*reinterpret_cast<const __half2*>(&vv.w));
      }
      float k0v = 0.0f;
      if (CH0 && (it.msk & 1u)) k0v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(st + S::R_K0)[j]);
      mbar_arrive(EMPTY(s));
      if (!valid) {
#pragma unroll
        for (int g = 0; g < kGroups; ++g) ksz[g] = vsz[g] = make_float2(0.0f, 0.0f);
        k0v = 0.0f;
      }
      // the value operand holds c - L/2, so the zero point carries the L/2 steps
      constexpr float kHalfL = ((1 << VB) - 1) * 0.5f;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) vsz[g].y = fmaf(kHalfL, vsz[g].x, vsz[g].y);

      ok &= ws_wait(SDONE(t % S::SB), (t / S::SB) & 1, err);
      tc_fence_after();
      float sc[HH];
      {
        // S_g = sum_c u8 code * (128 q1 + q2): q1 in column h, q2 in column G + h of group g
        uint32_t d1[kGroups][HH], d2[kGroups][HH];
        const uint32_t sbase = tmem + lane_base + S::TM_S + (t % S::SB) * 4 * S::NS + part * HH;
        if constexpr (HH == 2 || HH == 4) {
          tmem_ld8_wait<HH>(sbase, S::NS, G, d1, d2);
        } else {
          tmem_ld4_wait<HH>(sbase, S::NS, d1);
          tmem_ld4_wait<HH>(sbase + G, S::NS, d2);
        }
        const float* qsum = reinterpret_cast<const float*>(fix + S::F_QS + qb * G * 16);
        const float* q0s = reinterpret_cast<const float*>(fix + S::F_Q0 + qb * S::QV);
        const float* qds = reinterpret_cast<const float*>(fix + S::F_QD + qb * S::QV);
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const int hh = part * HH + i;
          float qg[kGroups], q0, qd;
          if constexpr (QREG) {
#pragma unroll
            for (int g = 0; g < kGroups; ++g) qg[g] = qsg[i][g];
            q0 = q0r[i];
            qd = qdr[i];
          } else {
            const float4 qs = reinterpret_cast<const float4*>(qsum)[hh];
            qg[0] = qs.x;
            qg[1] = qs.y;
            qg[2] = qs.z;
            qg[3] = qs.w;
            q0 = CH0 ? q0s[hh] : 0.0f;
            qd = qds[hh];
          }
          float dot = 0.0f, zt = CH0 ? q0 * k0v : 0.0f;
#pragma unroll
          for (int g = 0; g < kGroups; ++g) {
            const int dg = (int)d1[g][i] * 128 + (int)d2[g][i];  // exact: |dg| < 2^23
            dot = fmaf(ksz[g].x, (float)dg, dot);
            zt = fmaf(ksz[g].y, qg[g], zt);
          }
          sc[i] = fmaf(dot, qd, zt);
        }
      }
      tc_fence_before();
      if (it.last) mbar_arrive(QFREE(qb));  // done with this segment's query data and score UMMAs
      // lazy running max: raise it (part-wide) only if some score exceeds it by 2^kLazyMax
      bool exceed = false;
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        sc[i] = valid ? sc[i] * a.scale_log2 : NEG_INF;
        exceed |= sc[i] > m_run[i] + kLazyMax;
      }
      float* rt = red + (k * S::TPT + part) * 64;
      const bool raise = named_sync_or(bar_id, 128, exceed);
      if (raise) {  // uniform across the part
        float alpha[HH];
        float m_new[HH];
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const float mx = warp_max(sc[i]);
          if (lane == 0) rt[wq * 16 + i] = mx;
        }
        named_sync(bar_id, 128);
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          m_new[i] = fmaxf(m_run[i], fmaxf(fmaxf(rt[i], rt[16 + i]), fmaxf(rt[32 + i], rt[48 + i])));
          alpha[i] = exp2f(m_run[i] - m_new[i]);
          m_run[i] = m_new[i];
          l_acc[i] *= alpha[i];
#pragma unroll
          for (int g = 0; g < kGroups; ++g) zacc[g][i] *= alpha[i];
        }
        if (seg_tiles > 0) {
          // rescale the group's PV sums of the segment so far (this thread: channel
          // j, its heads) once the PV of its previous tile has landed; tile t's PV
          // adds after PREADY below
          ok &= ws_wait(PVDONE(last_own & 1), (last_own >> 1) & 1, err);
          tc_fence_after();
          const uint32_t base = obase(qb);
#pragma unroll
          for (int pp = 0; pp < PP; ++pp) {
            uint32_t r[HH];
            tmem_ld_wait<HH>(base + pp * S::NO, r);
#pragma unroll
            for (int i = 0; i < HH; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha[i]);
            tmem_st_n<HH>(base + pp * S::NO, r);
          }
          tmem_wait_st();
          tc_fence_before();
        }
      }
      float p[HH];
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        p[i] = valid ? exp2f(sc[i] - m_run[i]) : 0.0f;
        l_acc[i] += p[i];
#pragma unroll
        for (int g = 0; g < kGroups; ++g) zacc[g][i] = fmaf(p[i], vsz[g].y, zacc[g][i]);
      }
      // P' = p * value scale into the MN-major operand: column (group g, head),
      // K position pos.  This buffer was last read by the PV UMMAs of tile t-2.
      if (t >= 2) ok &= ws_wait(PVDONE(k), ((t - 2) >> 1) & 1, err);
      uint8_t* BP = fix + S::F_BP + k * S::BP_BYTES;
      if constexpr (G == 1) {
        // one head: columns 0..3 = groups 0..3, one 8-byte store
        const __half2 a01 = __floats2half2_rn(p[0] * vsz[0].x, p[0] * vsz[1].x);
        const __half2 a23 = __floats2half2_rn(p[0] * vsz[2].x, p[0] * vsz[3].x);
        *reinterpret_cast<uint2*>(BP + mnmajor(0, pos)) =
            make_uint2(*reinterpret_cast<const uint32_t*>(&a01), *reinterpret_cast<const uint32_t*>(&a23));
      } else if constexpr (S::TPT == 1) {
        // columns g*G + i, 0 .. 4G-1, contiguous: 8 per 16-byte store
        uint32_t pk[2 * G];
#pragma unroll
        for (int g = 0; g < kGroups; ++g)
#pragma unroll
          for (int i = 0; i < HH; i += 2) {
            const __half2 h2 = __floats2half2_rn(p[i] * vsz[g].x, p[i + 1] * vsz[g].x);
            pk[(g * HH + i) / 2] = *reinterpret_cast<const uint32_t*>(&h2);
          }
#pragma unroll
        for (int n = 0; n < 4 * G; n += 8)
          *reinterpret_cast<uint4*>(BP + mnmajor(n, pos)) =
              make_uint4(pk[n / 2], pk[n / 2 + 1], pk[n / 2 + 2], pk[n / 2 + 3]);
      } else {
        // HH consecutive columns g*G + part*HH .. per group
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
          uint32_t pk[HH / 2];
#pragma unroll
          for (int i = 0; i < HH; i += 2) {
            const __half2 h2 = __floats2half2_rn(p[i] * vsz[g].x, p[i + 1] * vsz[g].x);
            pk[i / 2] = *reinterpret_cast<const uint32_t*>(&h2);
          }
          uint8_t* dst = BP + mnmajor(g * G + part * HH, pos);
          if constexpr (HH == 2) *reinterpret_cast<uint32_t*>(dst) = pk[0];
          if constexpr (HH == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
          if constexpr (HH == 8) *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      fence_proxy_async();
      mbar_arrive(PREADY(k));
      ++seg_tiles;
      last_own = t;
      } else if (it.last) {
        mbar_arrive(QFREE(qb));  // done with this segment's query data
      }

      if (it.last && seg_tiles == 0) {
        // no tile of this segment fell to this group: an empty partial (the combine skips it)
        const int slot = ((int)it.bh(a) + blockIdx.x) * S::NGRP + grp;
        if (j == 0)
#pragma unroll
          for (int i = 0; i < HH; ++i) a.part_ml[(size_t)slot * G + part * HH + i] = make_float2(NEG_INF, 0.0f);
      } else if (it.last) {
        // segment totals over this part's 128 tokens (max, sum, value zero-point terms),
        // parked in shared memory until the segment's output is read out
        float* r2 = red2 + part * 64;
        float* pd = pend + (qb * S::TPT + part) * 6 * HH;
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const float sm = warp_sum(l_acc[i]);
          if (lane == 0) r2[wq * 16 + i] = sm;
        }
        named_sync(bar_id, 128);
        if (j == 0) {
#pragma unroll
          for (int i = 0; i < HH; ++i) {
            pd[i] = m_run[i];
            pd[HH + i] = r2[i] + r2[16 + i] + r2[32 + i] + r2[48 + i];
          }
        }
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
          named_sync(bar_id, 128);
#pragma unroll
          for (int i = 0; i < HH; ++i) {
            const float sm = warp_sum(zacc[g][i]);
            if (lane == 0) r2[wq * 16 + i] = sm;
          }
          named_sync(bar_id, 128);
          if (j == 0) {
#pragma unroll
            for (int i = 0; i < HH; ++i) pd[(2 + g) * HH + i] = r2[i] + r2[16 + i] + r2[32 + i] + r2[48 + i];
          }
        }
        named_sync(bar_id, 128);
        const int slot = ((int)it.bh(a) + blockIdx.x) * S::NGRP + grp;
        if (pn == 0) {
          p0_tile = last_own;
          p0_set = qb;
          p0_slot = slot;
        } else {
          p1_tile = last_own;
          p1_set = qb;
          p1_slot = slot;
        }
        ++pn;
      }
    }
    drain(ntiles + 2);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == S::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
}

// Merges a unit's partials (one per CTA its tiles were spread over) into one
// softmax over the whole sequence: o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s,
// rotated back into the value basis when the values were stored rotated.
__global__ void __launch_bounds__(kHeadDim) k_combine(DecodeArgs a, int G, int ngrp) {
  const int row = blockIdx.x;  // b * Hq + query head
  const int b = row / a.Hq, hq = row - b * a.Hq;
  const int h = hq / G, hl = hq - h * G;
  const int chn = threadIdx.x;
  int total = 0, tb = 0;
  for (int bb = 0; bb < a.c.B; ++bb) {
    if (bb == b) tb = total;
    total += a.c.H * tiles_of(a, bb);
  }
  const int nt = tiles_of(a, b);
  float out = 0.0f;
  if (nt > 0) {
    const int per = (total + kCtas - 1) / kCtas;
    const int u = b * a.c.H + h;
    const int tu = tb + h * nt;
    const int c0 = tu / per, c1 = (tu + nt - 1) / per;
    // slots (u + CTA) * ngrp + epilogue group; an empty one has max -inf and is skipped
    const float NEG_INF = -__int_as_float(0x7f800000);
    float M = NEG_INF;
    for (int sl = (u + c0) * ngrp; sl < (u + c1 + 1) * ngrp; ++sl) M = fmaxf(M, a.part_ml[(size_t)sl * G + hl].x);
    // the bf16 window tokens' partial, when the cache has windows
    const bool win = a.c.sink + a.c.recent > 0;
    const size_t rw = (size_t)(a.win_base + u) * G + hl;
    if (win) M = fmaxf(M, a.part_ml[rw].x);
    float l = 0.0f, o = 0.0f;
    for (int sl = (u + c0) * ngrp; sl < (u + c1 + 1) * ngrp + (win ? 1 : 0); ++sl) {
      const size_t r = sl < (u + c1 + 1) * ngrp ? (size_t)sl * G + hl : rw;
      const float2 v = a.part_ml[r];
      if (v.x == NEG_INF) continue;
      const float w = exp2f(v.x - M);
      l = fmaf(w, v.y, l);
      o = fmaf(w, a.part_acc[r * kHeadDim + chn], o);
    }
    out = o / l;
  }
  if (a.c.rotate_v) {
    // back from the rotated value basis: the orthonormal Walsh-Hadamard
    // transform is its own inverse (fp32 butterflies over the 128 channels)
    __shared__ float x[kHeadDim];
    x[chn] = out;
    for (int hs = 1; hs < kHeadDim; hs <<= 1) {
      __syncthreads();
      const float mine = x[chn], other = x[chn ^ hs];
      __syncthreads();
      x[chn] = (chn & hs) ? other - mine : mine + other;
    }
    __syncthreads();
    out = x[chn] * (float)a.inv_sqrt_d;
  }
  a.out[(size_t)row * kHeadDim + chn] = out;
}

template <int G, int KB, int VB, bool CH0, typename In>
cudaError_t launch_typed(const DecodeArgs& a, cudaStream_t s) {
  using S = Shape<G, KB, VB, CH0>;
  auto kern = k_decode<G, KB, VB, CH0, In>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<kCtas, S::THREADS, S::SMEM_BYTES, s>>>(a);
  return cudaGetLastError();
}

template <int G, int KB, int VB, bool CH0>
cudaError_t launch_dtype(const DecodeArgs& a, cudaStream_t s) {
  switch (a.dtype) {
    case KVQ_F32: return launch_typed<G, KB, VB, CH0, float>(a, s);
    case KVQ_BF16: return launch_typed<G, KB, VB, CH0, __nv_bfloat16>(a, s);
    default: return launch_typed<G, KB, VB, CH0, __half>(a, s);
  }
}

template <int KB, int VB, bool CH0>
cudaError_t launch_g(const DecodeArgs& a, cudaStream_t s) {
  switch (a.Hq / a.c.H) {
    case 1: return launch_dtype<1, KB, VB, CH0>(a, s);
    case 2: return launch_dtype<2, KB, VB, CH0>(a, s);
    case 4: return launch_dtype<4, KB, VB, CH0>(a, s);
    case 8: return launch_dtype<8, KB, VB, CH0>(a, s);
    case 16: return launch_dtype<16, KB, VB, CH0>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int KB, int VB>
cudaError_t launch_bits(const DecodeArgs& a, cudaStream_t s) {
  return a.c.keep_ch0 ? launch_g<KB, VB, true>(a, s) : launch_g<KB, VB, false>(a, s);
}

}  // namespace

bool decode_g_supported(int g) { return g == 1 || g == 2 || g == 4 || g == 8 || g == 16; }
int decode_groups(int) { return 1; }
int decode_slots(int B, int H, int G) { return (B * H + kCtas) * decode_groups(G); }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.c.k_bits == 4 && a.c.v_bits == 4) return launch_bits<4, 4>(a, s);
  if (a.c.k_bits == 4) return launch_bits<4, 2>(a, s);
  if (a.c.v_bits == 4) return launch_bits<2, 4>(a, s);
  return launch_bits<2, 2>(a, s);
}

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s) {
  k_combine<<<a.c.B * a.Hq, kHeadDim, 0, s>>>(a, a.Hq / a.c.H, decode_groups(a.Hq / a.c.H));
  return cudaGetLastError();
}

}  // namespace kvq
