// Split decode over the packed cache on the tcgen05 tensor cores: scores and
// the value sums are both integer MMAs straight from the codes.
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
// Per 128-token tile, 8 MMAs:
//   scores: 4 of kind::i8 (K = 32 = one quantization group each): key codes
//           as u8 in tensor memory x the rotated query as two exact s8 pieces
//           (q = delta_g * (128 q1 + q2), one step delta_g per channel group),
//           one s32 accumulator per group, so the per-token group scale and
//           the group's step apply exactly afterwards;
//   PV:     4 of kind::i8 (K = 32 tokens each): value codes as u8 in tensor
//           memory x P' as four u8 bytes of an integer up to 2^31, P' = p *
//           value scale normalized by running bounds (p relative to a lazily
//           raised running max, the scale relative to the running maximum
//           scale of its group), so the s32 sums are exact, P' never
//           overflows and keeps the 24 significant bits of the float it is
//           rounded from; each tile's sums are read back and added, with the
//           tile's scale, into fp32 accumulators held in registers.
//
// Roles inside a CTA, pipelined over tiles with mbarriers:
//   producer warps (2): 1-D bulk async copies of a tile's kept key-code rows
//                     (Dual-QK Sec. 3.3: channel-major rows, read selectively),
//                     value-code rows, key and value scale/zero pairs and
//                     channel 0 into one stage of a deep shared-memory ring;
//                     the two take alternate tiles;
//   code warps (4)  : thread = token: the token's key codes -> u8 -> tensor
//                     memory (lane = token); at a segment start also the
//                     query operand (dropped channel groups zeroed), its
//                     per-head step and its per-group sums; then, one tile
//                     behind, thread = channel: the channel's 128 value codes
//                     -> u8 -> tensor memory (lane = channel);
//   score warp      : the score MMAs, as far ahead as the score buffers allow;
//   PV warp         : the PV MMAs of each tile once its P' is written;
//   epilogue warps  : thread = (token, heads): score = sum_g delta_g s_g S_g +
//                     sum_g z_g sum(q_g) (+ q_0 k_0), the tile's maxima, the
//                     online softmax with a lazily raised running max, P' into
//                     shared memory, the value zero-point terms sum_t p_t z_t;
//                     thread = (channel, heads): the PV sums of an earlier
//                     tile into the fp32 accumulators.  Two epilogue groups
//                     take alternate tiles when the heads fit one thread.
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
constexpr float kLazyMax = 8.0f;  // the running max is raised only when a score exceeds it by 2^8 (log2 units)
constexpr int kMaxStages = 12;
constexpr int kSmemLimit = 227 * 1024;
constexpr float kQSteps = 16000.0f;  // |q| / delta <= 16000: pieces q1 in [-125, 125], q2 in [-64, 63]
// P' = p * value scale * 2^23 / vmr with p <= 2^kLazyMax and scale <= vmr, so
// P' <= 2^31: four u8 bytes, rounded from a float (24 significant bits)
constexpr float kPUnit = 8388608.0f;  // 2^23
constexpr int kProducers = 2;

template <int G, int KB, int VB, bool CH0>
struct Shape {
  static constexpr int TPT = G > 4 ? 2 : 1;  // epilogue threads per token (head parts)
  // epilogue groups: group g takes the tiles t with t % NGRP == g, so two
  // tiles' chains of waits and latencies overlap (as many as 16 warps allow)
  static constexpr int NGRP = TPT == 1 ? 2 : 1;
  static constexpr int HH = G / TPT;         // heads per epilogue thread: 1, 2, 4 or 8
  static constexpr int EPI_WARPS = 4 * TPT * NGRP;
  static constexpr int EPI_THREADS = 32 * EPI_WARPS;
  // two UMMA issuers: one thread can only have about one MMA in its issue
  // stage at a time (some 150 cycles each, whatever the shape), so the score
  // and the PV MMAs come from two warps and overlap
  static constexpr int MMA_WARP = 8 + EPI_WARPS;  // score MMAs
  static constexpr int PV_WARP = MMA_WARP + 1;    // PV MMAs
  // ring fillers: producer p issues the copies of the tiles t with t % NPROD == p
  // (a pruned tile takes one copy per run of kept channel groups)
  static constexpr int NPROD = kProducers;
  static constexpr int PROD_WARP = PV_WARP + 1;
  static constexpr int THREADS = 32 * (PROD_WARP + NPROD);
  // registers per thread: the block is launched with 65536 / THREADS; the
  // code warpgroups and the issue/producer warpgroup give some back to the
  // epilogue warpgroups (the shares add up to at most the launch total)
  static constexpr int REG_LAUNCH = 65536 / THREADS / 8 * 8;
  static constexpr int REG_KCODE = 80;
  static constexpr int REG_VCODE = 56;
  static constexpr int REG_ISSUE = 56;
  static constexpr int REG_REST = 128 * (REG_KCODE + REG_VCODE + REG_ISSUE);
  static constexpr int REG_EPI_FIT = (REG_LAUNCH * THREADS - REG_REST) / EPI_THREADS / 8 * 8;
  static constexpr int REG_EPI = REG_EPI_FIT > 248 ? 248 : REG_EPI_FIT;
  static_assert(THREADS == 256 + EPI_THREADS + 128, "warpgroups: key codes, value codes, epilogue, issue + producers");
  static_assert(REG_REST + EPI_THREADS * REG_EPI <= REG_LAUNCH * THREADS, "register split");
  static_assert(REG_EPI >= REG_LAUNCH, "register split");
  static constexpr int NS = 2 * G < 16 ? 16 : 2 * G;  // score columns per group: q1 rows, then q2 rows
  static constexpr int PH = 4 * G;  // P' columns per byte: (value group, head)
  static constexpr int KST = G > 8 ? 1 : 2;  // key operand stages in tensor memory
  static constexpr int VST = 2;              // value operand stages in tensor memory
  // PV columns: four bytes x (value group, head)
  static constexpr int NPV = 4 * PH;
  // score accumulator buffers: as many (up to 3) as leave room for two PV buffers
  static constexpr int SB = 128 + 3 * 4 * NS + 2 * NPV <= 512 ? 3 : (128 + 2 * 4 * NS + 2 * NPV <= 512 ? 2 : 1);
  static constexpr int NKR = KST > 1 ? KST : 2;  // key-ready barriers
  // tensor-memory columns
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_AK = 0;                 // KST key stages x 32 columns (128 u8 codes)
  static constexpr int TM_AV = 32 * KST;          // VST value stages x 32 columns (128 u8 codes)
  static constexpr int TM_S = 128;                // SB score buffers x 4 groups x NS
  static constexpr int TM_D = TM_S + SB * 4 * NS;  // DB PV buffers x NPV
  static constexpr int DB = TM_D + 2 * NPV <= TMEM_COLS ? 2 : 1;  // PV buffers: read back 2 or 1 tiles later
  static_assert(TM_AV + 32 * VST <= TM_S, "operand columns");
  static_assert(TM_D + DB * NPV <= TMEM_COLS, "tensor memory");
  static_assert(TM_S % NS == 0 && TM_D % NPV == 0, "accumulator alignment");
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
  static constexpr int BP_BYTES = NPV * kTile;       // one u8 P' operand: NPV columns x 128 tokens
  // query data per segment, double-buffered by segment parity
  static constexpr int QV = (G * 4 + 15) / 16 * 16;  // bytes of G floats, rounded to 16
  static constexpr int F_BQ = 0;                     // [2] query operands
  static constexpr int F_BP = F_BQ + 2 * BQ_BYTES;   // [2] P' buffers
  static constexpr int F_QS = F_BP + 2 * BP_BYTES;   // [2][G][4] f32: per-group sums of the kept q
  static constexpr int F_Q0 = F_QS + 2 * G * 16;     // [2][G] f32: q_0 (channel 0 kept in bf16)
  static constexpr int F_QD = F_Q0 + 2 * QV;         // [2][G][4] f32: step of the query pieces per group
  static constexpr int F_RED = F_QD + 2 * G * 16;  // [2 own tiles][NGRP][TPT][4 warps][16] s32: warp maxima
  static constexpr int F_RED2 = F_RED + 2 * NGRP * TPT * 4 * 16 * 4;  // [NGRP][TPT][4 warps][16] f32: segment sums
  static constexpr int F_BAR = (F_RED2 + NGRP * TPT * 4 * 16 * 4 + 15) / 16 * 16;
  // kready[3] vready[2] pready[2] sdone[3] pvdone[2] qready[2] qfree[2] sfree[3]
  static constexpr int NBAR_FIXED = 19;
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
// K position (byte) of token j of a tile in the u8 value operand: the INT4
// unpacking puts the even tokens of each 8-token word first, the INT2
// unpacking crumb m of every byte of a 16-token word together.
template <int BITS>
__device__ __forceinline__ int vpos_of(int j) {
  if (BITS == 4) return (j & ~7) + 4 * (j & 1) + ((j & 7) >> 1);
  return (j & ~15) + 4 * (j & 3) + ((j & 15) >> 2);
}
// byte offset of element (row r, byte k) in a K-major 8-bit operand with 128 K bytes
__device__ __forceinline__ uint32_t kmajor8(int r, int k) {
  return (r & 7) * 16 + (k & 15) + (k >> 4) * 128 + (r >> 3) * 1024;
}
// byte offset of element (n, k) in an MN-major 8-bit operand with 128 K elements
__device__ __forceinline__ uint32_t mnmajor8(int n, int k) {
  return (n & 15) + (k & 7) * 16 + (n >> 4) * 2048 + (k >> 3) * 128;
}
// Order-preserving map of a float onto int32 (and back: it is its own inverse),
// so that a warp's float maximum is one integer reduction.
__device__ __forceinline__ int ord_of(float x) {
  const int i = __float_as_int(x);
  return i >= 0 ? i : i ^ 0x7FFFFFFF;
}
__device__ __forceinline__ float float_of_ord(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7FFFFFFF); }

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
  if (__builtin_expect(mbar_test_wait(bar, parity), 1)) return true;
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
// Named barrier that also returns whether any participating thread passed true.
__device__ __forceinline__ bool bar_any(int id, int threads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
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
  constexpr int HH = S::HH, ST = S::STAGES;
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
  auto SFREE = [&](int k) { return bar0 + 8 * (16 + k); };   // the epilogue has read score buffer k
  auto FULL = [&](int s) { return bar0 + 8 * (S::NBAR_FIXED + s); };
  auto EMPTY = [&](int s) { return bar0 + 8 * (S::NBAR_FIXED + ST + s); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fix + S::F_SLOT);
  volatile int* err = reinterpret_cast<volatile int*>(fix + S::F_ERR);

  if (tid == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(FULL(s), 1);
      mbar_init(EMPTY(s), 256 + S::EPI_THREADS / S::NGRP);  // key and value conversion, the tile's epilogue group
    }
    for (int k = 0; k < S::NKR; ++k) mbar_init(KREADY(k), 128);
    for (int k = 0; k < S::SB; ++k) {
      mbar_init(SDONE(k), 1);
      mbar_init(SFREE(k), S::EPI_THREADS / S::NGRP);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(VREADY(k), 128);
      mbar_init(PREADY(k), S::EPI_THREADS / S::NGRP);
      mbar_init(PVDONE(k), 1);
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
  // Each warpgroup first sets its register budget (the code warps and the
  // issue/producer warpgroup give registers back to the epilogue), then
  // takes its role.
  if (warp < 4) {
    setmaxnreg_dec<S::REG_KCODE>();
    // ================================================================ key codes -> tensor memory
    // thread = token of the tile == tensor-memory lane of this warp's quarter
    const int j = tid;
    const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
    int kseg = 0;  // segments begun so far
    for (int t = 0; t < ntiles; ++t, it.next(a)) {
      const int s = t % ST;
      const uint8_t* raw = smem + s * S::STAGE + S::R_KC;
      ws_wait(FULL(s), (t / ST) & 1, err);
      // this key stage was read by the score UMMAs of tile t - KST
      if (t >= S::KST) ws_wait(SDONE((t - S::KST) % S::SB), ((t - S::KST) / S::SB) & 1, err);
      tc_fence_after();
      if (__builtin_expect(it.first, 0)) {
        // query data of segment kseg into buffer kseg & 1: per head and
        // 32-channel group g, delta_g = max|q_g| / 16000 and q = delta_g *
        // (128 q1 + q2) exactly (a step per group keeps a group of small
        // channels as fine as its own largest one allows); the rows of each
        // epilogue head part are its heads' q1 pieces, then their q2 pieces;
        // dropped channel groups (and channel 0 when it is kept in bf16) are zero.  The buffer was last used by segment kseg - 2, which the
        // epilogue (and so its score UMMAs) finished before freeing it.  Each
        // buffer's two barriers see one phase per use, in order, so no parity wait
        // can pass on a later or an earlier phase.
        const int qb = kseg & 1;
        if (kseg >= 2) ws_wait(QFREE(qb), ((kseg - 2) >> 1) & 1, err);
        uint8_t* BQ = fix + S::F_BQ + qb * S::BQ_BYTES;
        float* qsum = reinterpret_cast<float*>(fix + S::F_QS + qb * G * 16);
        float* q0s = reinterpret_cast<float*>(fix + S::F_Q0 + qb * S::QV);
        float* qds = reinterpret_cast<float*>(fix + S::F_QD + qb * G * 16);
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
          // the group's largest element: lanes 8g .. 8g + 7 hold group g
#pragma unroll
          for (int m = 1; m < 8; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, m));
          const float delta = amax > 0.0f ? amax / kQSteps : 1.0f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int ch = 4 * lane + i;
            const int qi = __float2int_rn(v[i] / delta);  // |qi| <= 16000
            const int q1 = (qi + 64) >> 7;                // nearest multiple of 128 below qi + 64
            const int q2 = qi - 128 * q1;                 // in [-64, 63]
            constexpr int blk = KB == 4 ? 8 : 16;
            const int p = (ch / blk) * blk + kpos_of<KB>(ch % blk);
            const int r1 = (hq / S::HH) * 2 * S::HH + hq % S::HH;
            BQ[kmajor8(r1, p)] = (uint8_t)(int8_t)q1;
            BQ[kmajor8(r1 + S::HH, p)] = (uint8_t)(int8_t)q2;
          }
#pragma unroll
          for (int m = 1; m < 8; m <<= 1) part += __shfl_xor_sync(kFull, part, m);
          if ((lane & 7) == 0) {
            qsum[hq * kGroups + (lane >> 3)] = part;
            qds[hq * kGroups + (lane >> 3)] = delta;
          }
          if (lane == 0) q0s[hq] = (CH0 && sel) ? x[0] : 0.0f;
        }
        fence_proxy_async();      // query operand (generic writes) -> tensor core
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
      tc_fence_before();
      mbar_arrive(KREADY(t % S::NKR));
      mbar_arrive(EMPTY(t % ST));
    }
  } else if (warp < 8) {
    setmaxnreg_dec<S::REG_VCODE>();
    // ================================================================ value codes -> tensor memory
    // thread = channel == tensor-memory lane of this warp's quarter
    const int j = tid - 128;
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    // the 16-byte chunks of a channel's value row are stored rotated by
    // channel, so the rows of 8 consecutive channels hit 8 different bank groups
    const int swz = VB == 4 ? (j >> 1) & 3 : (j >> 2) & 1;
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % ST;
      ws_wait(FULL(s), (t / ST) & 1, err);
      // this value stage was read by the PV UMMAs of tile t - VST
      if (t >= S::VST) ws_wait(PVDONE((t - S::VST) & 1), ((t - S::VST) >> 1) & 1, err);
      tc_fence_after();
      uint32_t r[32];
      const uint8_t* row = smem + s * S::STAGE + S::R_VC + j * S::VROW;
      if (VB == 4) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {  // 16-byte chunk k: tokens 32k .. 32k+31, 8 per word
          const uint4 w = *reinterpret_cast<const uint4*>(row + 16 * (k ^ swz));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            r[8 * k + 2 * i] = ws[i] & 0x0F0F0F0Fu;             // even tokens
            r[8 * k + 2 * i + 1] = (ws[i] >> 4) & 0x0F0F0F0Fu;  // odd tokens
          }
        }
      } else {
#pragma unroll
        for (int k = 0; k < 2; ++k) {  // 16-byte chunk k: tokens 64k .. 64k+63, 16 per word
          const uint4 w = *reinterpret_cast<const uint4*>(row + 16 * (k ^ swz));
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int m = 0; m < 4; ++m) r[16 * k + 4 * i + m] = (ws[i] >> (2 * m)) & 0x03030303u;
        }
      }
      const uint32_t vcol = tl + S::TM_AV + (t % S::VST) * 32;  // 128 u8 codes in the order vpos_of gives
      tmem_st16(vcol, *reinterpret_cast<const uint32_t(*)[16]>(&r[0]));
      tmem_st16(vcol + 16, *reinterpret_cast<const uint32_t(*)[16]>(&r[16]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(VREADY(t & 1));
      mbar_arrive(EMPTY(s));
    }
  } else if (warp < 8 + S::EPI_WARPS) {
    setmaxnreg_inc<S::REG_EPI>();
    // ================================================================ epilogue
    // With NGRP epilogue groups, group g takes the tiles t with t % NGRP == g;
    // each keeps its own online softmax and accumulators per segment and
    // leaves its own partial, which the combine merges like any other split.
    const int e = tid - 256;             // 0 .. EPI_THREADS-1
    const int grp = e / (128 * S::TPT);  // epilogue group
    const int j = e & 127;               // token (score phase) == tensor-memory lane == channel (PV phase)
    const int part = (e >> 7) % S::TPT;  // head part: heads part*HH .. part*HH + HH - 1
    const int wq = warp & 3;             // lane quarter == value group of channel j
    const int bar_id = 1 + grp * S::TPT + part;
    const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
    const int pos = vpos_of<VB>(j);      // K position of token j in the P' operand
    int* rmax = reinterpret_cast<int*>(fix + S::F_RED);  // [2][NGRP][TPT][16][4 warps]
    float* red2 = reinterpret_cast<float*>(fix + S::F_RED2) + (grp * S::TPT + part) * 64;  // [4][16]
    const float NEG_INF = -__int_as_float(0x7f800000);
    // P' columns: (part, group, head, byte), 16 HH per part; the four bytes of
    // one P' integer sit in adjacent columns, so a P' integer is one 32-bit word
    constexpr int NC = 16 * HH;
    const int n0 = part * NC;

    float m_run[HH], l_acc[HH], zacc[kGroups][HH];
    // running maximum of the value scales per group this segment, and 2^23 / it
    float vmr[kGroups], kvr[kGroups];
    float acc[HH];  // PV sums of channel j for this part's heads, scaled to m_run
    // PV sums of this group's last tile (ds1) and, when two of its tiles can be
    // in flight, the one before (ds2) still to be read back, with their scales
    // for channel j's group; tile t's sums sit in PV buffer t % DB and are read
    // back at tile t + DB, before the PV MMAs that reuse the buffer are issued
    constexpr int RD = S::DB;                // in tiles
    constexpr int PLEN = S::DB / S::NGRP;    // in this group's tiles: 1 or 2
    float ds1[HH] = {}, ds2[HH] = {};
    bool have1 = false, have2 = false;
    // this segment's query data for the thread's heads (per-group sums of the
    // kept q, q_0), held in registers when one thread takes a token's heads,
    // else read from shared memory per tile; the steps of the query pieces are
    // read from shared memory per tile
    constexpr bool QREG = S::TPT == 1;
    float qsg[QREG ? HH : 1][kGroups], q0r[QREG ? HH : 1];
    int nseg = 0;       // segments begun so far
    int qb = 0;         // query buffer of the current segment (its parity)
    int seg_tiles = 0;  // tiles of the current segment this group has taken
    int last_own = 0;   // the last tile this group took
    // where the bf16 windows sit for this segment's unit: the sequence position
    // of its token 0 and the length the windows are placed by (a bucket's
    // anchor and its sequence's length with bucket-relative RoPE)
    int wpos0 = 0, wlen = 0;
    bool ok = true;

    // add the PV sums of tile tp (buffer tp % DB) times its scale into acc:
    // the sums of the four bytes of P' (each exact in fp32)
    auto pv_addr = [&](int tp) { return tmem + lane_base + S::TM_D + (tp % S::DB) * S::NPV + n0 + wq * 4 * HH; };
    auto add_pv = [&](const uint32_t (&r)[4 * HH], const float (&ds)[HH]) {
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        float v = (float)(int)r[4 * i + 3];
        v = fmaf(v, 256.0f, (float)(int)r[4 * i + 2]);
        v = fmaf(v, 256.0f, (float)(int)r[4 * i + 1]);
        v = fmaf(v, 256.0f, (float)(int)r[4 * i]);
        acc[i] = fmaf(v, ds[i], acc[i]);
      }
    };
    auto read_pv = [&](int tp, const float (&ds)[HH]) {
      uint32_t r[4 * HH];  // (head, byte) of channel j's group
      tmem_ld_wait<4 * HH>(pv_addr(tp), r);
      add_pv(r, ds);
    };

    for (int t = 0; t < ntiles; ++t, it.next(a)) {
      const int k = t & 1;
      if (__builtin_expect(it.first, 0)) {
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          m_run[i] = NEG_INF;
          l_acc[i] = 0.0f;
          acc[i] = 0.0f;
#pragma unroll
          for (int g = 0; g < kGroups; ++g) zacc[g][i] = 0.0f;
        }
#pragma unroll
        for (int g = 0; g < kGroups; ++g) vmr[g] = kvr[g] = 0.0f;
        have1 = have2 = false;
        seg_tiles = 0;
        if (c.sink + c.recent > 0) {
          if (a.bucket_nb > 0) {
            wpos0 = (it.b % a.bucket_nb) * a.bucket_w;
            wlen = min(max(a.real_lens[it.b / a.bucket_nb], 0), a.real_max_len);
          } else {
            wpos0 = 0;
            wlen = it.len;
          }
        }
        qb = nseg & 1;  // this segment's query data
        ok &= ws_wait(QREADY(qb), (nseg >> 1) & 1, err);
        ++nseg;
        const float* qsum = reinterpret_cast<const float*>(fix + S::F_QS + qb * G * 16);
        const float* q0s = reinterpret_cast<const float*>(fix + S::F_Q0 + qb * S::QV);
#pragma unroll
        for (int i = 0; i < (QREG ? HH : 0); ++i) {
          const int hh = part * HH + i;
          const float4 qs = reinterpret_cast<const float4*>(qsum)[hh];
          qsg[i][0] = qs.x;
          qsg[i][1] = qs.y;
          qsg[i][2] = qs.z;
          qsg[i][3] = qs.w;
          q0r[i] = CH0 ? q0s[hh] : 0.0f;
        }
      }
      if (t % S::NGRP != grp) {
        if (it.last) mbar_arrive(QFREE(qb));  // done with this segment's query data
      } else {
      // tokens past the end, and the bf16 window tokens (scored by k_window), take no part
      const int tok = it.i * kTile + j;  // token position in the sequence
      const bool valid = tok < it.len && !in_window(c.sink, c.recent, wpos0 + tok, wlen);
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

      // The P' buffer k was read by the PV UMMAs of tile t - 2 (the UMMAs of
      // one thread complete in order, so PV t - 1 done implies PV t - 2 done),
      // whose sums, this group's when it has one in this segment, are read back
      // before the running max can move.  With one epilogue group, tile t - 2
      // is two tiles back and long done: its sums come in the same
      // tensor-memory round trip as the scores.  With two, it is this group's
      // previous tile, still in flight: they come after the scores.
      constexpr bool MERGED = HH <= 4 && S::NGRP == 1;
      ok &= ws_wait(SDONE(t % S::SB), (t / S::SB) & 1, err);
      if (MERGED && t >= RD) ok &= ws_wait(PVDONE((t - RD) & 1), ((t - RD) >> 1) & 1, err);
      const bool rdp = t >= RD && (PLEN == 2 ? have2 : have1);
      tc_fence_after();
      // S_g = sum_c u8 code * (128 q1 + q2): q1 in column 2 HH part + h, q2 in
      // column 2 HH part + HH + h of group g
      uint32_t sd[kGroups][2 * HH];
      const uint32_t sbase = tmem + lane_base + S::TM_S + (t % S::SB) * 4 * S::NS + part * 2 * HH;
      if constexpr (HH <= 4) {
        tmem_ld4_wait<2 * HH>(sbase, S::NS, sd);
        tc_fence_before();
      } else {
        uint32_t d1[kGroups][HH], d2[kGroups][HH];
        tmem_ld4_wait<HH>(sbase, S::NS, d1);
        tmem_ld4_wait<HH>(sbase + HH, S::NS, d2);
#pragma unroll
        for (int g = 0; g < kGroups; ++g)
#pragma unroll
          for (int i = 0; i < HH; ++i) {
            sd[g][i] = d1[g][i];
            sd[g][HH + i] = d2[g][i];
          }
        tc_fence_before();
      }
      float sc[HH];
      {
        const float* qsum = reinterpret_cast<const float*>(fix + S::F_QS + qb * G * 16);
        const float* q0s = reinterpret_cast<const float*>(fix + S::F_Q0 + qb * S::QV);
        const float* qds = reinterpret_cast<const float*>(fix + S::F_QD + qb * G * 16);
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const int hh = part * HH + i;
          float qg[kGroups], q0;
          const float4 qd = reinterpret_cast<const float4*>(qds)[hh];  // the head's steps per group
          const float qdg[kGroups] = {qd.x, qd.y, qd.z, qd.w};
          if constexpr (QREG) {
#pragma unroll
            for (int g = 0; g < kGroups; ++g) qg[g] = qsg[i][g];
            q0 = q0r[i];
          } else {
            const float4 qs = reinterpret_cast<const float4*>(qsum)[hh];
            qg[0] = qs.x;
            qg[1] = qs.y;
            qg[2] = qs.z;
            qg[3] = qs.w;
            q0 = CH0 ? q0s[hh] : 0.0f;
          }
          // dot and zero-point sums over the groups as one paired fma each
          float2 dz = make_float2(0.0f, CH0 ? q0 * k0v : 0.0f);
#pragma unroll
          for (int g = 0; g < kGroups; ++g) {
            const int dg = (int)sd[g][i] * 128 + (int)sd[g][HH + i];  // exact: |dg| < 2^23
            dz = ffma2(ksz[g], make_float2((float)dg * qdg[g], qg[g]), dz);
          }
          sc[i] = valid ? (dz.x + dz.y) * a.scale_log2 : NEG_INF;
        }
      }
      mbar_arrive(SFREE(t % S::SB));        // the score buffer may take tile t + SB
      if (it.last) mbar_arrive(QFREE(qb));  // done with this segment's query data and score UMMAs

      // P' is normalized by running bounds, not by the tile's own maxima:
      // scores count from the running max m_run, raised only when a score
      // passes it by 2^kLazyMax, and value scales from the running maximum vmr
      // of their group.  One barrier with an OR tells the part whether any of
      // its tokens passes a bound; only then are the tile's maxima reduced.
      bool pass = false;
#pragma unroll
      for (int i = 0; i < HH; ++i) pass |= sc[i] > m_run[i] + kLazyMax;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) pass |= vsz[g].x > vmr[g];
      // with the sums of tile t - RD long done, their load is in flight while
      // the part's warps meet at the barrier
      uint32_t pv[4 * HH];
      if constexpr (MERGED) {
        tc_fence_after();
        tmem_ld_start<4 * HH>(pv_addr(t), pv);
      }
      const bool raise = bar_any(bar_id, 128, pass);
      if constexpr (MERGED) {
        tmem_ld_finish<4 * HH>(pv);
        tc_fence_before();
        if (rdp) add_pv(pv, PLEN == 2 ? ds2 : ds1);
      }
      float alpha[HH];
      if (__builtin_expect(raise, 0)) {
        // the tile's largest score per head and largest value scale per group
        // (warp maxima, then the part's four warps through shared memory)
        int* rk = rmax + ((((t / S::NGRP) & 1) * S::NGRP + grp) * S::TPT + part) * 64;
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const int m = __reduce_max_sync(kFull, ord_of(sc[i]));
          if (lane == 0) rk[4 * i + wq] = m;
        }
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {  // scales are >= 0: their bits order like the values
          const unsigned m = __reduce_max_sync(kFull, __float_as_uint(vsz[g].x));
          if (lane == 0) rk[4 * (HH + g) + wq] = (int)m;
        }
        named_sync(bar_id, 128);
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const int4 w = reinterpret_cast<const int4*>(rk)[i];
          const float smax = float_of_ord(max(max(w.x, w.y), max(w.z, w.w)));
          const float m_new = fmaxf(m_run[i], smax);
          alpha[i] = m_new == NEG_INF ? 1.0f : exp2f(m_run[i] - m_new);
          m_run[i] = m_new;
        }
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
          const int4 w = reinterpret_cast<const int4*>(rk)[HH + g];
          vmr[g] = fmaxf(vmr[g], __uint_as_float((unsigned)max(max(w.x, w.y), max(w.z, w.w))));
          kvr[g] = vmr[g] > 0.0f ? __fdividef(kPUnit, vmr[g]) : 0.0f;
        }
      }

      if (!MERGED && t >= RD) {
        ok &= ws_wait(PVDONE((t - RD) & 1), ((t - RD) >> 1) & 1, err);
        if (rdp) {
          tc_fence_after();
          read_pv(t, PLEN == 2 ? ds2 : ds1);  // tile t - RD, in PV buffer (t - RD) % DB = t % DB
          tc_fence_before();
        }
      }
      if (__builtin_expect(raise, 0)) {
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          l_acc[i] *= alpha[i];
          acc[i] *= alpha[i];
          ds1[i] *= alpha[i];
#pragma unroll
          for (int g = 0; g < kGroups; ++g) zacc[g][i] *= alpha[i];
        }
      }
      // p = 2^(s - m_run) in [0, 2^kLazyMax]; P' = p * scale * 2^23 / vmr rounded
      // to an integer in [0, 2^31]
      float pn[HH];
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        pn[i] = valid ? exp2f(sc[i] - m_run[i]) : 0.0f;
        l_acc[i] += pn[i];
      }
      uint32_t xw[kGroups * HH];  // column order: group, then head
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
        const float vk = vsz[g].x * kvr[g];
        if constexpr (HH == 1) {
          zacc[g][0] = fmaf(pn[0], vsz[g].y, zacc[g][0]);
          xw[g] = __float2uint_rn(pn[0] * vk);
        } else {
#pragma unroll
          for (int i = 0; i < HH; i += 2) {  // heads in pairs: one paired fma per pair
            const float2 z = ffma2(make_float2(pn[i], pn[i + 1]), make_float2(vsz[g].y, vsz[g].y),
                                   make_float2(zacc[g][i], zacc[g][i + 1]));
            zacc[g][i] = z.x;
            zacc[g][i + 1] = z.y;
            xw[g * HH + i] = __float2uint_rn(pn[i] * vk);
            xw[g * HH + i + 1] = __float2uint_rn(pn[i + 1] * vk);
          }
        }
      }
      // the tile's PV sums (read back RD tiles later) carry vmr / 2^23 for
      // channel j's group
      float ds0[HH];
#pragma unroll
      for (int i = 0; i < HH; ++i) ds0[i] = vmr[wq] * (1.0f / kPUnit);
      // four P' words (16 columns, one 16-byte row of the operand) per store
      uint8_t* BP = fix + S::F_BP + k * S::BP_BYTES;
#pragma unroll
      for (int w = 0; w < kGroups * HH / 4; ++w)
        *reinterpret_cast<uint4*>(BP + mnmajor8(n0 + 16 * w, pos)) =
            make_uint4(xw[4 * w], xw[4 * w + 1], xw[4 * w + 2], xw[4 * w + 3]);
      fence_proxy_async();
      mbar_arrive(PREADY(k));
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        ds2[i] = ds1[i];
        ds1[i] = ds0[i];
      }
      have2 = PLEN == 2 && have1;
      have1 = true;
      ++seg_tiles;
      last_own = t;
      }  // own tile

      if (__builtin_expect(it.last && seg_tiles == 0, 0)) {
        // no tile of this segment fell to this group: an empty partial (the combine skips it)
        const int slot = ((int)it.bh(a) + blockIdx.x) * S::NGRP + grp;
        if (j == 0)
#pragma unroll
          for (int i = 0; i < HH; ++i)
            if (kvq_in_bounds((size_t)slot * G + part * HH + i, 1, a.part_rows))
              a.part_ml[(size_t)slot * G + part * HH + i] = make_float2(NEG_INF, 0.0f);
      } else if (__builtin_expect(it.last, 0)) {
        // this group's pending PV sums of the segment, then its totals over the
        // tokens (max, sum, value zero-point terms) into its partial slot
        const int tl1 = last_own, tl2 = last_own - S::NGRP;  // its last tile, and the one before
        if (PLEN == 2 && have2) {
          ok &= ws_wait(PVDONE(tl2 & 1), (tl2 >> 1) & 1, err);
          tc_fence_after();
          read_pv(tl2, ds2);
        }
        ok &= ws_wait(PVDONE(tl1 & 1), (tl1 >> 1) & 1, err);
        tc_fence_after();
        read_pv(tl1, ds1);
        tc_fence_before();
        have1 = have2 = false;
        const int slot = ((int)it.bh(a) + blockIdx.x) * S::NGRP + grp;
        const float nan = __int_as_float(0x7fc00000);
        const bool good = ok && !*err;
        float lsum[HH];
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const float sm = warp_sum(l_acc[i]);
          if (lane == 0) red2[wq * 16 + i] = sm;
        }
        named_sync(bar_id, 128);
#pragma unroll
        for (int i = 0; i < HH; ++i) lsum[i] = red2[i] + red2[16 + i] + red2[32 + i] + red2[48 + i];
        float zown[HH];  // sum over the tokens of p * zero of channel j's group
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
          named_sync(bar_id, 128);
#pragma unroll
          for (int i = 0; i < HH; ++i) {
            const float sm = warp_sum(zacc[g][i]);
            if (lane == 0) red2[wq * 16 + i] = sm;
          }
          named_sync(bar_id, 128);
          if (g == wq) {
#pragma unroll
            for (int i = 0; i < HH; ++i) zown[i] = red2[i] + red2[16 + i] + red2[32 + i] + red2[48 + i];
          }
        }
        named_sync(bar_id, 128);
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const size_t row = (size_t)slot * G + part * HH + i;
          if (!kvq_in_bounds(row, 1, a.part_rows)) continue;
          a.part_acc[row * kHeadDim + j] = good ? acc[i] + zown[i] : nan;
          if (j == 0) a.part_ml[row] = good ? make_float2(m_run[i], lsum[i]) : make_float2(nan, nan);
        }
      }
    }
  } else {
    setmaxnreg_dec<S::REG_ISSUE>();
    if (warp == S::MMA_WARP) {
      // ================================================================ score UMMAs
      // As far ahead as the SB score buffers allow: buffer t % SB was last read
      // by the epilogue of tile t - SB, which frees it (SFREE) once its scores are
      // in registers.
      const uint32_t idesc_s = idesc_u8s8_s32(kTile, S::NS);
      int sseg = -1;  // segment of the tile being scored
      for (int t = 0; t < ntiles; ++t, it.next(a)) {
        if (it.first) ++sseg;
        const uint32_t bq = smem_addr(fix + S::F_BQ + (sseg & 1) * S::BQ_BYTES);
        if (t >= S::SB) ws_wait(SFREE(t % S::SB), ((t - S::SB) / S::SB) & 1, err);
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
      }
    } else if (warp == S::PV_WARP) {
      // ================================================================ PV UMMAs
      const uint32_t idesc_o = idesc_u8u8_s32_bmn(kTile, S::NPV);
      const uint32_t bp = smem_addr(fix + S::F_BP);
      for (int t = 0; t < ntiles; ++t) {
        ws_wait(PREADY(t & 1), (t >> 1) & 1, err);
        ws_wait(VREADY(t & 1), (t >> 1) & 1, err);
        tc_fence_after();
        if (lane == 0) {
          // 32 tokens per MMA: u8 value codes (8 tensor-memory columns) x the
          // tile's P' bytes; each tile's sums start afresh in PV buffer t % DB
          const uint32_t a0 = tmem + S::TM_AV + (t % S::VST) * 32;
          const uint32_t b0 = bp + (t & 1) * S::BP_BYTES;
          const uint32_t d0 = tmem + S::TM_D + (t % S::DB) * S::NPV;
  #pragma unroll
          for (int s = 0; s < kTile / 32; ++s)
            umma_i8_tmem_a(d0, a0 + s * 8, smem_desc(b0 + s * 512, 128, 2048), idesc_o, s > 0 ? 1u : 0u);
          umma_commit(PVDONE(t & 1));
        }
        __syncwarp();
      }
    } else {
      // ================================================================ producers
      const int nblk = c.cap / kTile;
      const int pw = warp - S::PROD_WARP;
      for (int t = 0; t < ntiles; ++t, it.next(a)) {
        if (t % S::NPROD != pw) continue;
        // test hook: leave this tile's stage unfilled, so that the waits on it give up
        if (blockIdx.x == 0 && t == a.withheld_tile) continue;
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
        // (a copy the bounds checks refuse leaves its stage short: its waits give up)
        if (run_start) {
          const int run = __ffsll((long long)~((unsigned long long)msk >> lane)) - 1;
          const size_t off = key_word_index(bh, c.cap, lane, n0) * (KB == 4 ? 2 : 1);
          if (kvq_in_bounds(off, run * S::KROW, c.kc_bytes()))
            bulk_g2s(dst + S::R_KC + lane * S::KROW, c.kc + off, run * S::KROW, FULL(s));
        }
        if (lane == 0 && kvq_in_bounds(blk * kHeadDim * S::VROW, kHeadDim * S::VROW, c.vc_bytes()))
          bulk_g2s(dst + S::R_VC, c.vc + blk * kHeadDim * S::VROW, kHeadDim * S::VROW, FULL(s));
        if (lane == 1 && kvq_in_bounds(key_scale_index(bh, c.cap, 0, n0), kGroups * kTile, c.ks_pairs()))
          bulk_g2s(dst + S::R_KS, c.ks + key_scale_index(bh, c.cap, 0, n0), kGroups * kTile * 4, FULL(s));
        if (lane == 2 && kvq_in_bounds((bh * c.cap + n0) * kGroups, kTile * kGroups, c.ks_pairs()))
          bulk_g2s(dst + S::R_VS, c.vs + (bh * c.cap + n0) * kGroups, kTile * kGroups * 4, FULL(s));
        if (k0 && lane == 3 && kvq_in_bounds(bh * c.cap + n0, kTile, c.rows()))
          bulk_g2s(dst + S::R_K0, c.k0 + bh * c.cap + n0, kTile * 2, FULL(s));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*err) {
    // a wait gave up: copies and MMAs issued before it may still be in flight;
    // let them land (they take microseconds) before the tensor memory is freed
    // and the CTA exits, and report the give-up to the host
#pragma unroll 1
    for (int i = 0; i < 64; ++i) __nanosleep(1000);
    if (tid == 0 && a.status) atomicOr(a.status, 1);
  }
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
  // tiles of the whole batch and of the sequences before b (block-wide sums)
  const int2 tp = block_tile_prefix(a.c.B, b, a.c.H, [&](int bb) { return tiles_of(a, bb); });
  const int total = tp.x, tb = tp.y;
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
    for (int sl = (u + c0) * ngrp; sl < (u + c1 + 1) * ngrp; ++sl)
      if (kvq_in_bounds((size_t)sl * G + hl, 1, a.part_rows)) M = fmaxf(M, a.part_ml[(size_t)sl * G + hl].x);
    // the bf16 window tokens' partial, when the cache has windows
    const bool win = a.c.sink + a.c.recent > 0;
    const size_t rw = (size_t)(a.win_base + u) * G + hl;
    if (win && kvq_in_bounds(rw, 1, a.part_rows)) M = fmaxf(M, a.part_ml[rw].x);
    float l = 0.0f, o = 0.0f;
    for (int sl = (u + c0) * ngrp; sl < (u + c1 + 1) * ngrp + (win ? 1 : 0); ++sl) {
      const size_t r = sl < (u + c1 + 1) * ngrp ? (size_t)sl * G + hl : rw;
      if (!kvq_in_bounds(r, 1, a.part_rows)) continue;
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
int decode_groups(int G) { return G <= 4 ? 2 : 1; }
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

KVQ_BOUNDS_COUNTER(bounds_decode)

}  // namespace kvq

