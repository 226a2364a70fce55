// Persistent, warp-specialized split decode on the tcgen05 tensor cores.
//
// Work split ("stream-K"): every (sequence b, kv head h) unit contributes
// ceil(len_b / 128) tiles; the tiles of all units, in (b, h) order, are cut
// into 148 equal contiguous ranges, one per CTA (one CTA per SM).  A CTA's
// range covers one or more unit segments; each segment leaves one partial
// (running max, sum, accumulator per query head) in slot (unit + CTA), a slot
// index that is unique because consecutive units' CTA ranges only touch at
// their ends.  The combine pass merges a unit's slots into one softmax over
// the whole sequence (Dual-QK summary Sec. 3.4).
//
// Roles inside a CTA (18 warps), pipelined across tiles with mbarriers:
//   producer warp : 1-D bulk async copies of each tile's raw key-code rows (kept
//                   channel groups only) and value codes into a 3-deep ring,
//                   and of its per-token scales, zeros and channel 0 into a
//                   4-deep ring;
//   converter warps (8): key codes -> exact f16 integers, tile AK (K-major,
//                   token x channel); value codes -> tile AV (MN-major,
//                   channel x token); at a segment start also the query
//                   operand (rotated q as f16 hi/lo) and its per-group sums;
//   UMMA warp     : score UMMAs (one f32 accumulator per 32-channel group, so
//                   per-token group scales apply exactly afterwards; q's f16
//                   hi and lo parts accumulate into the same column) one tile
//                   ahead, then the PV UMMAs O[channel][group x head];
//   epilogue warps (4 per 4 heads): thread = (token, 4 heads): scores from
//                   tensor memory, s_g * dot + z_g * sum(q) (+ q_0 k_ch0), the
//                   online softmax with a lazily raised max, P' = p * value
//                   scale_g into tile BP, the value zero-point term and sums in
//                   registers; one tile later, thread = (channel, 4 heads): O
//                   from tensor memory into a rescaled register accumulator;
//                   at a segment end, the partial.
// Scores come straight from the codes; no dequantized key is ever formed
// (tq-kv abstract; Dual-QK summary Sec. 3.2, 3.3).  Every mbarrier wait is
// bounded; after a give-up all waits fall through and the CTA writes NaN
// partials instead of hanging.
#include "common.cuh"
#include "sm100.cuh"

namespace kvq {
namespace {

using namespace sm100;

constexpr int kWsCtas = 148;  // one persistent CTA per SM
constexpr int kTile = 128;
constexpr int kConvWarps = 8;   // warps 0-3 convert key codes, warps 4-7 value codes
constexpr int kKWarps = 4;
constexpr int kOBufs = 3;       // PV accumulators in flight (read back two tiles late)
constexpr float kLazyMax = 8.0f;  // the running max is raised only when a score exceeds it by 2^8
constexpr int kRing = 2;                                       // raw code stages
constexpr int kSRing = 3;                                      // per-token scale/zero stages

template <int G, int KB, int VB, bool CH0>
struct WsShape {
  static constexpr int TPT = G >= 8 ? 2 : 1;          // epilogue threads per token (head parts)
  static constexpr int EPI_WARPS = 4 * TPT;
  static constexpr int MMA_WARP = kConvWarps + EPI_WARPS;
  static constexpr int PROD_WARP = MMA_WARP + 1;
  static constexpr int THREADS = (PROD_WARP + 1) * 32;
  static constexpr int NS = G < 16 ? 16 : G;          // score columns per group: one per head (zero pad)
  static constexpr int NO = 4 * G;                    // PV columns: group x head
  static constexpr int HH = G / TPT;                  // heads per epilogue thread
  static constexpr int TM_S = 0;                      // two score buffers of 4 * NS columns
  static constexpr int TM_O = 2 * 4 * NS;             // kOBufs PV buffers of NO columns
  static constexpr int TMEM_COLS = (TM_O + kOBufs * NO) <= 256 ? 256 : 512;
  static constexpr int KW = KB == 4 ? 2 : 1;
  static constexpr int KROW = kTile * KW;
  static constexpr int VROW = kHeadDim * VB / 8;
  static constexpr int TILE_AB = kTile * kHeadDim * 2;  // one f16 operand tile
  static constexpr int KW_ = KB == 4 ? 2 : 1;
  static constexpr int RAW_BYTES_ = kPruneGroups * kTile * KW_ + kTile * (kHeadDim * VB / 8);
  // key operand stages: three when they fit next to everything else, else two
  static constexpr int KST = (3 * TILE_AB + 2 * TILE_AB + 4 * NS * kHeadDim + 2 * NO * kTile * 2 +
                              kRing * RAW_BYTES_ + kSRing * (kTile * kGroups * 8 + kTile * 2) + 2048) <= 227 * 1024
                                 ? 3 : 2;
  static constexpr int AK_OFF = 0;
  static constexpr int AV_OFF = AK_OFF + KST * TILE_AB;
  static constexpr int BQ_OFF = AV_OFF + 2 * TILE_AB;
  static constexpr int BQ_HALF = NS * kHeadDim * 2;    // q hi rows, then q lo rows
  static constexpr int BQ_BYTES = 2 * BQ_HALF;
  static constexpr int BP_OFF = BQ_OFF + BQ_BYTES;
  static constexpr int BP_BYTES = NO * kTile * 2;
  static constexpr int RAW_OFF = BP_OFF + 2 * BP_BYTES;
  static constexpr int R_KC = 0;
  static constexpr int R_VC = kPruneGroups * KROW;
  static constexpr int RAW_BYTES = R_VC + kTile * VROW;
  // scale ring: key (scale, zero) [4 groups][128 tokens], value (scale, zero)
  // [128 tokens][4 groups], channel 0 [128 tokens]
  static constexpr int SC_OFF = RAW_OFF + kRing * RAW_BYTES;
  static constexpr int S_KS = 0;
  static constexpr int S_VS = S_KS + kGroups * kTile * 4;
  static constexpr int S_K0 = S_VS + kTile * kGroups * 4;
  static constexpr int SC_BYTES = S_K0 + (CH0 ? kTile * 2 : 0);
  static constexpr int QSUM_OFF = SC_OFF + kSRing * SC_BYTES;   // [G][4] f32
  static constexpr int Q0_OFF = QSUM_OFF + G * kGroups * 4;     // [G] f32
  static constexpr int RED_OFF = Q0_OFF + G * 4;                // [2 tiles][2 parts][4 warps][8] f32
  static constexpr int RED2_OFF = RED_OFF + 2 * 2 * 4 * 8 * 4;  // [2 parts][4 warps][8] f32 (segment sums)
  // segment results waiting for their last PV: [2 tile parities][2 parts] x (max[4], sum[4], zero term[4 groups][4])
  static constexpr int PEND_OFF = RED2_OFF + 2 * 4 * 8 * 4;
  static constexpr int PEND_BYTES = 2 * 2 * 24 * 4;
  static constexpr int BAR_OFF = PEND_OFF + PEND_BYTES;
  // mbarriers: full[R], empty[R], kready[2], vready[2], pready[2], sdone[3], pvdone[3],
  // sfull[SR], sempty[SR]
  static constexpr int NBAR = 2 * kRing + 12 + 2 * kSRing;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;
  static constexpr int ERR_OFF = SLOT_OFF + 4;
  static constexpr int SMEM_BYTES = ERR_OFF + 12;
};

template <int BITS>
__device__ __forceinline__ int ws_pos_of(int i) {
  if (BITS == 4) return i < 4 ? 2 * i : 2 * (i - 4) + 1;
  return i < 8 ? 2 * i : 2 * (i - 8) + 1;
}
template <int BITS>
__device__ __forceinline__ int ws_chan_of(int p) {
  if (BITS == 4) return (p & ~7) + ((p & 7) >> 1) + 4 * (p & 1);
  return (p & ~15) + ((p & 15) >> 1) + 8 * (p & 1);
}
__device__ __forceinline__ uint32_t ws_kmajor(int r, int k) {
  return (r & 7) * 16 + (k & 7) * 2 + (k >> 3) * 128 + (r >> 3) * 2048;
}
__device__ __forceinline__ uint32_t ws_mnmajor(int mn, int k) {
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
  int g, g_end, b, h, i, tiles_b, len, seg;
  uint32_t msk;  // kept channel groups of the current unit
  bool first, last;

  __device__ void load_mask(const DecodeArgs& a) { msk = a.mask ? a.mask[(size_t)b * a.c.H + h] : kFull; }

  __device__ void init(const DecodeArgs& a, int g0, int g1) {
    g = g0;
    g_end = g1;
    seg = 0;
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
    if (first) {
      ++seg;
      load_mask(a);
    }
    last = (i == tiles_b - 1) || (g == g_end - 1);
  }
  __device__ size_t bh(const DecodeArgs& a) const { return (size_t)b * a.c.H + h; }
};

// Bounded wait.  After a few quick polls the thread backs off with nanosleep
// (32 ns doubling to 256 ns), so waiting warps leave the issue slots to the
// warps doing work; it gives up after ~2^22 polls (about a second), or at once
// after any earlier give-up in the CTA.
__device__ __forceinline__ bool ws_wait(uint32_t bar, uint32_t parity, volatile int* err) {
#pragma unroll 1
  for (int i = 0; i < 4; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  unsigned ns = 32;
#pragma unroll 1
  for (uint32_t it = 0; it < (1u << 22); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*err) return false;
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
  }
  *err = 1;
  return false;
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <int G, int KB, int VB, bool CH0, typename In>
__global__ void __launch_bounds__(WsShape<G, KB, VB, CH0>::THREADS, 1) k_decode_split_ws(DecodeArgs a) {
  using S = WsShape<G, KB, VB, CH0>;
  constexpr int HH = S::HH;
  static_assert(HH == 4, "epilogue packs 4 heads per thread; slot 7 of each reduction row is a flag");
  constexpr int EPI_THREADS = S::EPI_WARPS * 32;
  extern __shared__ __align__(1024) uint8_t smem[];
  const CacheView& c = a.c;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- this CTA's tile range
  int total = 0;
  for (int b = 0; b < c.B; ++b) total += c.H * tiles_of(a, b);
  const int per = (total + kWsCtas - 1) / kWsCtas;
  const int g0 = blockIdx.x * per, g1 = min(g0 + per, total);
  if (g0 >= g1) return;
  const int ntiles = g1 - g0;

  const uint32_t bar0 = smem_addr(smem + S::BAR_OFF);
  auto FULL = [&](int s) { return bar0 + 8 * s; };
  auto EMPTY = [&](int s) { return bar0 + 8 * (kRing + s); };
  auto KREADY = [&](int k) { return bar0 + 8 * (2 * kRing + k); };
  auto VREADY = [&](int k) { return bar0 + 8 * (2 * kRing + 2 + k); };
  auto PREADY = [&](int k) { return bar0 + 8 * (2 * kRing + 4 + k); };
  auto SDONE = [&](int k) { return bar0 + 8 * (2 * kRing + 6 + k); };   // k < KST: one per key stage
  auto PVDONE = [&](int k) { return bar0 + 8 * (2 * kRing + 9 + k); };  // k < kOBufs
  auto SFULL = [&](int s) { return bar0 + 8 * (2 * kRing + 12 + s); };
  auto SEMPTY = [&](int s) { return bar0 + 8 * (2 * kRing + 12 + kSRing + s); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::SLOT_OFF);
  volatile int* err = reinterpret_cast<volatile int*>(smem + S::ERR_OFF);

  if (tid == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(FULL(s), 1);
      mbar_init(EMPTY(s), kConvWarps * 32);
    }
    for (int s = 0; s < kSRing; ++s) {
      mbar_init(SFULL(s), 1);
      mbar_init(SEMPTY(s), EPI_THREADS);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(KREADY(k), kKWarps * 32);
      mbar_init(VREADY(k), (kConvWarps - kKWarps) * 32);
      mbar_init(PREADY(k), EPI_THREADS);
    }
    for (int k = 0; k < S::KST; ++k) mbar_init(SDONE(k), 1);
    for (int k = 0; k < kOBufs; ++k) mbar_init(PVDONE(k), 1);
    *err = 0;
    mbar_fence_init();
  }
  if (warp == S::MMA_WARP) {
    tmem_alloc(smem_addr(tmem_slot), S::TMEM_COLS);
    tmem_relinquish();
  }
  for (int i = tid; i < S::BQ_BYTES / 16; i += S::THREADS)
    reinterpret_cast<uint4*>(smem + S::BQ_OFF)[i] = make_uint4(0, 0, 0, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  TileIter it;
  it.init(a, g0, g1);

  if (warp == S::PROD_WARP) {
    // ================================================================ producer
    for (int t = 0; t < ntiles; ++t, it.next(a)) {
      const int s = t % kRing;
      if (t >= kRing) ws_wait(EMPTY(s), ((t / kRing) - 1) & 1, err);
      const size_t bh = it.bh(a);
      const uint32_t msk = it.msk;
      const int n0 = it.i * kTile;
      constexpr int ntc = kTile;  // cap and n0 are multiples of the 128-token key block
      const uint32_t dst = smem_addr(smem + S::RAW_OFF + s * S::RAW_BYTES);
      if (lane == 0) mbar_arrive_expect_tx(FULL(s), (uint32_t)(__popc(msk) * ntc * S::KW + ntc * S::VROW));
      __syncwarp();
      // one copy per run of adjacent kept channel groups (their rows are adjacent in the block)
      const bool run_start = ((msk >> lane) & 1u) && (lane == 0 || !((msk >> (lane - 1)) & 1u));
      if (run_start) {
        const int run = __ffsll((long long)~((unsigned long long)msk >> lane)) - 1;
        bulk_g2s(dst + S::R_KC + lane * S::KROW, c.kc + key_word_index(bh, c.cap, lane, n0) * S::KW,
                 run * ntc * S::KW, FULL(s));
      }
      if (lane == 0) bulk_g2s(dst + S::R_VC, c.vc + (bh * c.cap + n0) * S::VROW, ntc * S::VROW, FULL(s));
      // per-token scales and zeros (and channel 0) for the epilogue
      const int ss = t % kSRing;
      if (t >= kSRing) ws_wait(SEMPTY(ss), ((t / kSRing) - 1) & 1, err);
      const uint32_t sdst = smem_addr(smem + S::SC_OFF + ss * S::SC_BYTES);
      const bool k0 = CH0 && (msk & 1u);
      if (lane == 0)
        mbar_arrive_expect_tx(SFULL(ss), (uint32_t)(kGroups * ntc * 4 + ntc * 16 + (k0 ? ntc * 2 : 0)));
      __syncwarp();
      if (lane == kGroups + 2)  // the block's 4 scale rows are contiguous
        bulk_g2s(sdst + S::S_KS, c.ks + key_scale_index(bh, c.cap, 0, n0), kGroups * ntc * 4, SFULL(ss));
      if (lane == kGroups) bulk_g2s(sdst + S::S_VS, c.vs + (bh * c.cap + n0) * kGroups, ntc * 16, SFULL(ss));
      if (k0 && lane == kGroups + 1) bulk_g2s(sdst + S::S_K0, c.k0 + bh * c.cap + n0, ntc * 2, SFULL(ss));
    }
  } else if (warp == S::MMA_WARP) {
    // ================================================================ UMMA issue
    const uint32_t idesc_s = idesc_f16_f32(kTile, S::NS, 0, 0);
    const uint32_t idesc_o = idesc_f16_f32(kTile, S::NO, 1, 1);
    const uint32_t ak = smem_addr(smem + S::AK_OFF), av = smem_addr(smem + S::AV_OFF);
    const uint32_t bq = smem_addr(smem + S::BQ_OFF), bp = smem_addr(smem + S::BP_OFF);
    auto score = [&](int t) {
      ws_wait(KREADY(t & 1), (t >> 1) & 1, err);
      if (lane == 0) {
        tc_fence_after();
        const uint32_t a0 = ak + (t % S::KST) * S::TILE_AB, b0 = bq;
        // descriptors advance by 256 B (16 channels) per step: +16 in the 16-byte address field
        const uint64_t da = smem_desc(a0, 128, 2048), db = smem_desc(b0, 128, 2048);
#pragma unroll
        for (int step = 0; step < 4 * kGroups; ++step) {
          // group g: its 32 channels against q hi (part 0), then q lo (part 1), summed by the tensor core
          const int g = step >> 2, part = (step >> 1) & 1, s = step & 1, ks = 2 * g + s;
          umma_f16(tmem + S::TM_S + (t & 1) * 4 * S::NS + g * S::NS, da + (uint64_t)(ks * 16),
                   db + (uint64_t)((part * S::BQ_HALF + ks * 256) >> 4), idesc_s, (part | s) ? 1u : 0u);
        }
        umma_commit(SDONE(t % S::KST));
      }
      __syncwarp();
    };
    score(0);
    for (int t = 0; t < ntiles; ++t) {
      if (t + 1 < ntiles) score(t + 1);
      ws_wait(PREADY(t & 1), (t >> 1) & 1, err);
      ws_wait(VREADY(t & 1), (t >> 1) & 1, err);
      if (lane == 0) {
        tc_fence_after();
        const uint32_t a0 = av + (t & 1) * S::TILE_AB, b0 = bp + (t & 1) * S::BP_BYTES;
        const uint64_t da = smem_desc(a0, 128, 2048), db = smem_desc(b0, 128, 2048);
#pragma unroll
        for (int s = 0; s < kTile / 16; ++s)
          umma_f16(tmem + S::TM_O + (t % kOBufs) * S::NO, da + (uint64_t)(s * 16), db + (uint64_t)(s * 16), idesc_o,
                   s > 0 ? 1u : 0u);
        umma_commit(PVDONE(t % kOBufs));
      }
      __syncwarp();
    }
  } else if (warp < kKWarps) {
    // ================================================================ key converters
    const int j = tid & 127;  // token of the tile
    for (int t = 0; t < ntiles; ++t, it.next(a)) {
      const int s = t % kRing, k = t & 1;
      const uint8_t* raw = smem + S::RAW_OFF + s * S::RAW_BYTES;
      const size_t bh = it.bh(a);
      const uint32_t msk = it.msk;
      const int ks = t % S::KST;
      ws_wait(FULL(s), (t / kRing) & 1, err);
      // AK[ks] was read by the score UMMAs of tile t - KST
      if (t >= S::KST) ws_wait(SDONE(ks), ((t - S::KST) / S::KST) & 1, err);
      if (it.first) {
        // query operand of the new segment: BQ (hi, lo), per-group sums and q_0.  The
        // previous tile's epilogue (and so its score UMMAs) must be done with the old ones.
        if (t >= 1) ws_wait(PREADY((t - 1) & 1), ((t - 1) >> 1) & 1, err);
        uint8_t* BQ = smem + S::BQ_OFF;
        float* qsum = reinterpret_cast<float*>(smem + S::QSUM_OFF);
        float* q0s = reinterpret_cast<float*>(smem + S::Q0_OFF);
        for (int hq = warp; hq < G; hq += kKWarps) {
          const In* qrow = static_cast<const In*>(a.q) + ((size_t)it.b * a.Hq + (size_t)it.h * G + hq) * kHeadDim;
          float x[4];
          load_row_warp(qrow, c.rotate != 0, a.inv_sqrt_d, lane, x);
          const bool sel = (msk >> lane) & 1u;
          float part = 0.0f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int ch = 4 * lane + i;
            float v = sel ? x[i] : 0.0f;
            if (CH0 && ch == 0) v = 0.0f;
            part += v;
            const __half hi = __float2half_rn(v);
            const __half lo = __float2half_rn(v - __half2float(hi));
            const int blk = KB == 4 ? 8 : 16;
            const int p = (ch / blk) * blk + ws_pos_of<KB>(ch % blk);
            *reinterpret_cast<__half*>(BQ + ws_kmajor(hq, p)) = hi;
            *reinterpret_cast<__half*>(BQ + S::BQ_HALF + ws_kmajor(hq, p)) = lo;
          }
#pragma unroll
          for (int m = 1; m < 8; m <<= 1) part += __shfl_xor_sync(kFull, part, m);
          if ((lane & 7) == 0) qsum[hq * kGroups + (lane >> 3)] = part;
          if (lane == 0) q0s[hq] = (CH0 && sel) ? x[0] : 0.0f;
        }
      }
      // key codes -> AK[k]: every word is read (rows of dropped groups hold stale
      // codes) and dropped groups are zeroed by a select, so the loads issue
      // back to back with no branches between them
      uint8_t* AK = smem + S::AK_OFF + ks * S::TILE_AB;
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        if (KB == 4) {
          const uint16_t* kc = reinterpret_cast<const uint16_t*>(raw + S::R_KC) + j;
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = kc[(hh * 16 + i) * kTile];
#pragma unroll
          for (int qq = 0; qq < 8; ++qq) {
            const int q = hh * 8 + qq;
            const uint32_t w0 = ((msk >> (2 * q)) & 1u) ? w[2 * qq] : 0u;
            const uint32_t w1 = ((msk >> (2 * q + 1)) & 1u) ? w[2 * qq + 1] : 0u;
            uint32_t r[4];
            codes4_to_f16(w0 | (w1 << 16), r);
            *reinterpret_cast<uint4*>(AK + ws_kmajor(j, 8 * q)) = make_uint4(r[0], r[1], r[2], r[3]);
          }
        } else {
          const uint8_t* kc = raw + S::R_KC + j;
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = kc[(hh * 16 + i) * kTile];
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int q = hh * 4 + qq;
            uint32_t x = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) x |= (((msk >> (4 * q + i)) & 1u) ? w[4 * qq + i] : 0u) << (8 * i);
            uint32_t r[8];
            codes2_to_f16(x, r);
            *reinterpret_cast<uint4*>(AK + ws_kmajor(j, 16 * q)) = make_uint4(r[0], r[1], r[2], r[3]);
            *reinterpret_cast<uint4*>(AK + ws_kmajor(j, 16 * q + 8)) = make_uint4(r[4], r[5], r[6], r[7]);
          }
        }
      }
      fence_proxy_async();
      mbar_arrive(KREADY(k));
      mbar_arrive(EMPTY(s));
    }
  } else if (warp < kConvWarps) {
    // ================================================================ value converters
    const int j = tid & 127;  // token of the tile
    for (int t = 0; t < ntiles; ++t) {
      const int s = t % kRing, k = t & 1;
      const uint8_t* raw = smem + S::RAW_OFF + s * S::RAW_BYTES;
      ws_wait(FULL(s), (t / kRing) & 1, err);
      if (t >= 2) ws_wait(PVDONE((t - 2) % kOBufs), ((t - 2) / kOBufs) & 1, err);  // AV[k] read by PV of t-2
      uint8_t* AV = smem + S::AV_OFF + k * S::TILE_AB;
      constexpr int CHUNKS = S::VROW / 16;  // 16-byte chunks of a value row: 4 (INT4) or 2 (INT2)
#pragma unroll 1
      for (int r2 = 0; r2 < CHUNKS; ++r2) {
        // rotate the chunk order across tokens so each 8-thread phase reads 8 distinct banks
        const int kk = VB == 4 ? (r2 ^ ((j >> 1) & 3)) : (r2 ^ ((j >> 2) & 1));
        const uint4 w = *reinterpret_cast<const uint4*>(raw + S::R_VC + j * S::VROW + kk * 16);
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          if (VB == 4) {
            uint32_t r[4];
            codes4_to_f16(ws[i], r);
            *reinterpret_cast<uint4*>(AV + ws_mnmajor(8 * (4 * kk + i), j)) = make_uint4(r[0], r[1], r[2], r[3]);
          } else {
            uint32_t r[8];
            codes2_to_f16(ws[i], r);
            const int p = 64 * kk + 16 * i;
            *reinterpret_cast<uint4*>(AV + ws_mnmajor(p, j)) = make_uint4(r[0], r[1], r[2], r[3]);
            *reinterpret_cast<uint4*>(AV + ws_mnmajor(p + 8, j)) = make_uint4(r[4], r[5], r[6], r[7]);
          }
        }
      }
      fence_proxy_async();
      mbar_arrive(VREADY(k));
      mbar_arrive(EMPTY(s));
    }
  } else {
    // ================================================================ epilogue
    const int e = tid - kConvWarps * 32;  // 0 .. EPI_THREADS-1
    const int j = e & 127;                // token (score phase) == tensor-memory lane == channel position (PV)
    const int part = e >> 7;              // head part: heads part*HH .. part*HH + HH - 1
    const int wq = warp & 3;              // lane quarter == channel group in the PV phase
    const int bar_id = 1 + part;          // named barrier of this part's 4 warps
    const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
    float* red = reinterpret_cast<float*>(smem + S::RED_OFF);    // [2][2][4][8]
    float* red2 = reinterpret_cast<float*>(smem + S::RED2_OFF);  // [2][4][8]
    const int ch = ws_chan_of<VB>(j);

    float m_run[HH], l_acc[HH], zacc[kGroups][HH], o[HH];
    float qs_reg[kGroups][HH], q0_reg[HH];
    // per-tile rescale factors and segment flags of the two tiles whose PV is still pending
    float alpha1[HH], alpha2[HH];
    bool first1 = false, last1 = false, first2 = false, last2 = false;
    int slot_even = 0, slot_odd = 0;  // partial slot of a segment ending at an even / odd tile
    float* pend = reinterpret_cast<float*>(smem + S::PEND_OFF);  // [parity][part][24]
    bool ok = true;
#pragma unroll
    for (int i = 0; i < HH; ++i) {
      m_run[i] = -__int_as_float(0x7f800000);
      l_acc[i] = 0.0f;
      o[i] = 0.0f;
      alpha1[i] = alpha2[i] = 0.0f;
      q0_reg[i] = 0.0f;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) zacc[g][i] = qs_reg[g][i] = 0.0f;
    }

    // PV of tile tp into o (thread = channel position j); at a segment end, the partial
    auto readback = [&](int tp, const float (&alpha)[HH], bool first, bool last) {
      ok &= ws_wait(PVDONE(tp % kOBufs), (tp / kOBufs) & 1, err);
      tc_fence_after();
      uint32_t d[HH];
      tmem_ld<HH>(tmem + lane_base + S::TM_O + (tp % kOBufs) * S::NO + wq * G + part * HH, d);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < HH; ++i) o[i] = first ? __uint_as_float(d[i]) : fmaf(o[i], alpha[i], __uint_as_float(d[i]));
      tc_fence_before();
      if (last) {
        const float nan = __int_as_float(0x7fc00000);
        const bool good = ok && !*err;
        const float* pd = pend + ((tp & 1) * 2 + part) * 24;
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const size_t row = (size_t)((tp & 1) ? slot_odd : slot_even) * G + part * HH + i;
          a.part_acc[row * kHeadDim + ch] = good ? o[i] + pd[8 + wq * 4 + i] : nan;
          if (j == 0) a.part_ml[row] = good ? make_float2(pd[i], pd[4 + i]) : make_float2(nan, nan);
        }
      }
    };

    for (int t = 0; t < ntiles; ++t, it.next(a)) {
      const int k = t & 1;
      const size_t bh = it.bh(a);
      const uint32_t msk = it.msk;
      const int n0 = it.i * kTile;
      const bool valid = n0 + j < it.len;
      if (it.first) {
        // new segment: fresh softmax state
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          m_run[i] = -__int_as_float(0x7f800000);
          l_acc[i] = 0.0f;
#pragma unroll
          for (int g = 0; g < kGroups; ++g) zacc[g][i] = 0.0f;
        }
      }
      // per-token scales, zeros and channel 0 from the scale ring
      const int ss = t % kSRing;
      ok &= ws_wait(SFULL(ss), (t / kSRing) & 1, err);
      const uint8_t* sc_st = smem + S::SC_OFF + ss * S::SC_BYTES;
      float2 ksz[kGroups], vsz[kGroups];
#pragma unroll
      for (int g = 0; g < kGroups; ++g)
        ksz[g] = __half22float2(reinterpret_cast<const __half2*>(sc_st + S::S_KS + g * kTile * 4)[j]);
      {
        const uint4 vv = reinterpret_cast<const uint4*>(sc_st + S::S_VS)[j];
        vsz[0] = __half22float2(*reinterpret_cast<const __half2*>(&vv.x));
        vsz[1] = __half22float2(*reinterpret_cast<const __half2*>(&vv.y));
        vsz[2] = __half22float2(*reinterpret_cast<const __half2*>(&vv.z));
        vsz[3] = __half22float2(*reinterpret_cast<const __half2*>(&vv.w));
      }
      float k0v = 0.0f;
      if (CH0 && (msk & 1u)) k0v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(sc_st + S::S_K0)[j]);
      mbar_arrive(SEMPTY(ss));

      ok &= ws_wait(SDONE(t % S::KST), (t / S::KST) & 1, err);
      tc_fence_after();
      if (it.first) {
        // the segment's query sums: written by the converters before the score UMMAs of
        // this tile were issued, so visible once those completed
        const float* qsum = reinterpret_cast<const float*>(smem + S::QSUM_OFF);
        const float* q0s = reinterpret_cast<const float*>(smem + S::Q0_OFF);
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          q0_reg[i] = q0s[part * HH + i];
#pragma unroll
          for (int g = 0; g < kGroups; ++g) qs_reg[g][i] = qsum[(part * HH + i) * kGroups + g];
        }
      }
      float sc[HH];
#pragma unroll
      for (int i = 0; i < HH; ++i) sc[i] = CH0 ? q0_reg[i] * k0v : 0.0f;
      {
        uint32_t d[kGroups][HH];
#pragma unroll
        for (int g = 0; g < kGroups; ++g)
          tmem_ld<HH>(tmem + lane_base + S::TM_S + k * 4 * S::NS + g * S::NS + part * HH, d[g]);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < kGroups; ++g)
#pragma unroll
          for (int i = 0; i < HH; ++i)
            sc[i] = fmaf(ksz[g].x, __uint_as_float(d[g][i]), fmaf(ksz[g].y, qs_reg[g][i], sc[i]));
      }
      tc_fence_before();
      // lazy running max: raise it (CTA-part-wide) only if some score exceeds it by 2^kLazyMax
      bool exceed = false;
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        sc[i] = valid ? sc[i] * a.scale_log2 : -__int_as_float(0x7f800000);
        exceed |= sc[i] > m_run[i] + kLazyMax;
      }
      float* rt = red + (k * 2 + part) * 32;
      const unsigned any = __any_sync(kFull, exceed);
      if (lane == 0) rt[wq * 8 + 7] = any ? 1.0f : 0.0f;
      named_sync(bar_id, 128);
      const bool raise = (rt[7] + rt[15] + rt[23] + rt[31]) > 0.0f;
      float m_new[HH];
      if (raise) {  // uniform across the part
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const float mx = warp_max(sc[i]);
          if (lane == 0) rt[wq * 8 + i] = mx;
        }
        named_sync(bar_id, 128);
#pragma unroll
        for (int i = 0; i < HH; ++i)
          m_new[i] = fmaxf(m_run[i], fmaxf(fmaxf(rt[i], rt[8 + i]), fmaxf(rt[16 + i], rt[24 + i])));
      } else {
#pragma unroll
        for (int i = 0; i < HH; ++i) m_new[i] = m_run[i];
      }
      float alpha[HH];
      uint32_t pk[kGroups][HH / 2];
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        alpha[i] = exp2f(m_run[i] - m_new[i]);
        m_run[i] = m_new[i];
        const float p = valid ? exp2f(sc[i] - m_new[i]) : 0.0f;
        sc[i] = p;
        l_acc[i] = fmaf(l_acc[i], alpha[i], p);
#pragma unroll
        for (int g = 0; g < kGroups; ++g) zacc[g][i] = fmaf(zacc[g][i], alpha[i], p * vsz[g].y);
      }
#pragma unroll
      for (int g = 0; g < kGroups; ++g)
#pragma unroll
        for (int i = 0; i < HH; i += 2) {
          const __half2 h2 = __floats2half2_rn(sc[i] * vsz[g].x, sc[i + 1] * vsz[g].x);
          pk[g][i / 2] = *reinterpret_cast<const uint32_t*>(&h2);
        }
      uint8_t* BP = smem + S::BP_OFF + k * S::BP_BYTES;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) {
        const int n = g * G + part * HH;
#pragma unroll
        for (int i = 0; i < HH; i += 4)
          *reinterpret_cast<uint2*>(BP + ws_mnmajor(n + i, j)) = make_uint2(pk[g][i / 2], pk[g][i / 2 + 1]);
      }
      fence_proxy_async();
      mbar_arrive(PREADY(k));

      if (t >= 2) readback(t - 2, alpha2, first2, last2);
#pragma unroll
      for (int i = 0; i < HH; ++i) {
        alpha2[i] = alpha1[i];
        alpha1[i] = alpha[i];
      }
      first2 = first1;
      last2 = last1;
      first1 = it.first;
      last1 = it.last;

      if (it.last) {
        // segment totals over this part's 128 tokens (max, sum, value zero-point terms),
        // parked in shared memory until the segment's last PV is read back
        float* r2 = red2 + part * 32;
        float* pd = pend + ((t & 1) * 2 + part) * 24;
#pragma unroll
        for (int i = 0; i < HH; ++i) {
          const float s = warp_sum(l_acc[i]);
          if (lane == 0) r2[wq * 8 + i] = s;
        }
        named_sync(bar_id, 128);
        if (j == 0) {
#pragma unroll
          for (int i = 0; i < HH; ++i) {
            pd[i] = m_run[i];
            pd[4 + i] = r2[i] + r2[8 + i] + r2[16 + i] + r2[24 + i];
          }
        }
#pragma unroll
        for (int g = 0; g < kGroups; ++g) {
          named_sync(bar_id, 128);
#pragma unroll
          for (int i = 0; i < HH; ++i) {
            const float s = warp_sum(zacc[g][i]);
            if (lane == 0) r2[wq * 8 + i] = s;
          }
          named_sync(bar_id, 128);
          if (j == 0) {
#pragma unroll
            for (int i = 0; i < HH; ++i) pd[8 + g * 4 + i] = r2[i] + r2[8 + i] + r2[16 + i] + r2[24 + i];
          }
        }
        named_sync(bar_id, 128);
        if (t & 1)
          slot_odd = (int)bh + blockIdx.x;
        else
          slot_even = (int)bh + blockIdx.x;
      }
    }
    if (ntiles >= 2) readback(ntiles - 2, alpha2, first2, last2);
    readback(ntiles - 1, alpha1, first1, last1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == S::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
}

__global__ void __launch_bounds__(kHeadDim) k_combine_ws(DecodeArgs a, int G) {
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
    const int per = (total + kWsCtas - 1) / kWsCtas;
    const int u = b * a.c.H + h;
    const int tu = tb + h * nt;
    const int c0 = tu / per, c1 = (tu + nt - 1) / per;
    float M = -__int_as_float(0x7f800000);
    for (int cc = c0; cc <= c1; ++cc) M = fmaxf(M, a.part_ml[(size_t)(u + cc) * G + hl].x);
    float l = 0.0f, o = 0.0f;
    for (int cc = c0; cc <= c1; ++cc) {
      const size_t r = (size_t)(u + cc) * G + hl;
      const float2 v = a.part_ml[r];
      const float w = exp2f(v.x - M);
      l = fmaf(w, v.y, l);
      o = fmaf(w, a.part_acc[r * kHeadDim + chn], o);
    }
    out = o / l;
  }
  a.out[(size_t)row * kHeadDim + chn] = out;
}

template <int G, int KB, int VB, bool CH0, typename In>
cudaError_t launch_ws_typed(const DecodeArgs& a, cudaStream_t s) {
  using S = WsShape<G, KB, VB, CH0>;
  static_assert(S::SMEM_BYTES <= 227 * 1024, "shared memory");
  auto kern = k_decode_split_ws<G, KB, VB, CH0, In>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  kern<<<kWsCtas, S::THREADS, S::SMEM_BYTES, s>>>(a);
  return cudaGetLastError();
}

template <int G, int KB, int VB, bool CH0>
cudaError_t launch_ws_dtype(const DecodeArgs& a, cudaStream_t s) {
  switch (a.dtype) {
    case KVQ_F32: return launch_ws_typed<G, KB, VB, CH0, float>(a, s);
    case KVQ_BF16: return launch_ws_typed<G, KB, VB, CH0, __nv_bfloat16>(a, s);
    default: return launch_ws_typed<G, KB, VB, CH0, __half>(a, s);
  }
}

template <int KB, int VB, bool CH0>
cudaError_t launch_ws_g(const DecodeArgs& a, cudaStream_t s) {
  switch (a.Hq / a.c.H) {
    case 4: return launch_ws_dtype<4, KB, VB, CH0>(a, s);
    case 8: return launch_ws_dtype<8, KB, VB, CH0>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int KB, int VB>
cudaError_t launch_ws_bits(const DecodeArgs& a, cudaStream_t s) {
  return a.c.keep_ch0 ? launch_ws_g<KB, VB, true>(a, s) : launch_ws_g<KB, VB, false>(a, s);
}

}  // namespace

bool decode_ws_supported(int g) { return g == 4 || g == 8; }
int decode_ws_slots(int B, int H) { return B * H + kWsCtas; }

cudaError_t launch_decode_split_ws(const DecodeArgs& a, cudaStream_t s) {
  if (a.c.k_bits == 4 && a.c.v_bits == 4) return launch_ws_bits<4, 4>(a, s);
  if (a.c.k_bits == 4) return launch_ws_bits<4, 2>(a, s);
  if (a.c.v_bits == 4) return launch_ws_bits<2, 4>(a, s);
  return launch_ws_bits<2, 2>(a, s);
}

cudaError_t launch_combine_ws(const DecodeArgs& a, cudaStream_t s) {
  k_combine_ws<<<a.c.B * a.Hq, kHeadDim, 0, s>>>(a, a.Hq / a.c.H);
  return cudaGetLastError();
}

}  // namespace kvq
