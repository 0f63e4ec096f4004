// Block-causal multi-scale attention on tcgen05 tensor cores (sm_100a):
//   * S-CAS calibration attention (vark_scas_accumulate): queries of scale k
//     attend to every key of scales 0..k, and the softmax probability mass each
//     query row puts on each source scale is reduced per (head, s, k).
//     [HeatKV] project page, Method step 2 (attention aggregated per layer,
//     head, source scale and future scale) and step 3 (S-CAS).
//   * Pruned-cache attention (vark_pruned_attention): queries of scale k attend
//     to their head's retained past scales (compacted, ragged per head) and to
//     their own scale from the dense cache.  [HeatKV] Method step 5; [AMS-KV]
//     Abstract (the local scale is always attended).
//
// One CTA computes two 128-row query tiles (A, B) of the same (batch, head,
// query scale): they see the same key list, so every K/V tile is loaded once
// for 256 query rows.  Roles (384 threads, 3 warpgroups):
//   warp 0       TMA producer: Q_A, Q_B, then K and V tiles into 2-stage rings
//                with separate release points for K (after both S MMAs) and V
//                (after both PV MMAs);
//   warp 1       owns TMEM (512 columns) and issues tcgen05.mma from one
//                thread, ping-ponging the tiles: PV_A(j-1), S_A(j), PV_B(j-1),
//                S_B(j) -- so the softmax of one tile overlaps the other
//                tile's two MMAs;
//   warps 4-7    softmax of tile A, warps 8-11 softmax of tile B: one thread per
//                query row (TMEM lane = row).  S_X is read with tcgen05.ld, the
//                online softmax runs in the exp2 domain, and P_X is written back
//                as bf16 over the first 64 columns of S_X, where the PV MMA reads
//                it as its A operand straight from tensor memory.  O_X is
//                rescaled in TMEM only when a row's max grows by more than 2^8
//                (the stale max cancels in O / l).
// TMEM: S_A [0,128) S_B [128,256) O_A [256,256+D) O_B [256+D,256+2D).
// Shared memory: Q_A, Q_B, K and V rings, 128-byte swizzled (Q, K K-major; V
// MN-major as stored, [key][d]).  setmaxnreg moves registers from the control
// warpgroup to the two softmax warpgroups.
// Every mbarrier wait is bounded: on timeout the kernel records
// VARK_E_TIMEOUT in the caller's status word, drains its own async work with
// bounded waits, frees TMEM and returns.
#include <algorithm>
#include <cstdlib>
#include <vector>

#include "vark_common.cuh"

namespace vark {
namespace attn {

constexpr int kThreads = 384;
constexpr int kBlockM = 128;
constexpr int kBlockN = 128;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxPairs = 512;
constexpr int kMaxDesc = 256;            // key tiles with a precomputed descriptor
// (batch, head) blocks interleaved in the launch order: pruned attention
// gains from ending each launch on light CTAs; calibration, whose per-head
// K/V is larger, measured best head by head.
template <bool PRUNED>
struct HeadGroup { static constexpr int value = PRUNED ? 8 : 1; };
constexpr int kPanelBytes = 128 * 128;   // 128 rows x 128 bytes (64 bf16)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 domain
// Of every 8 columns of a full single-segment tile, this many take 2^x from the
// FMA-pipe polynomial and the rest from MUFU ex2.  With O the tile period is set
// by the S -> P -> PV -> S chain together with the MMA issuer's bookkeeping,
// not by MUFU throughput: shares of 2, 4, 6 per 8 ran 5-17% slower than 0,
// so the polynomial path is off.
constexpr int kPolyPer8 = 0;
// Without an output (S-CAS only) there is no P -> PV -> S chain and the
// softmax is bound by MUFU throughput: there 2 of 8 columns on the polynomial
// measured 12% faster than 0 (4 of 8: 7%).
constexpr int kPolyPer8NoO = 2;
// Columns of a full tile exponentiated against the running max before the
// tile max is known (calibration with O, after the first tile).
constexpr int kSpecKeys = 64;
template <int N>
struct Int { static constexpr int value = N; };


struct Params {
  ScaleTable sc;
  int B, H;
  int n_pairs;                    // query-tile pairs per (batch, head)
  uint32_t pair[kMaxPairs];       // (scale << 24) | first row of tile A within the scale
  float scale_log2;               // log2(e) / sqrt(D)
  const float* tau;
  const float* bias;              // [H][S] or null
  float* mass;                    // [H][S][S] (calibration)
  uint16_t* out;                  // same layout as q, or null
  int32_t* status;
  int q_rows;                     // rows per (b, h) of q / out
  int q_scale_rows;               // 1: q row = row within scale (single-scale q)
  int local_scale_only;           // 1: the local K/V source holds only the query scale's rows
  // pruned attention
  int64_t R_l;
  const int32_t* head_off;        // [H]
  const int32_t* seg_off;         // [H][S]
  const int32_t* past_len;        // [H][S]
  // packed retained past (pruned attention over a quantised cache): this
  // layer's codes ([kc_rows][D * bits / 8] bytes, K and V) and per-(batch,
  // head, scale, channel) tables [B][H][S][D] (8-bit: fp32 absmax; 4- and
  // 3-bit: bf16 scale bits); null otherwise
  const void* kq;
  const void* vq;
  const void* ktab;
  const void* vtab;
  int64_t kc_rows;                // rows of the compacted layout (bounds of the code reads)
  // failure-detection test hook (off by default): wait limit, and a key tile
  // the producer withholds so that waits on it run out
  uint64_t wait_limit_ns;
  int withhold_tile;
};

// P_X is written and consumed in kPChunks column chunks of kBlockN / kPChunks
// keys: the softmax stores a chunk as soon as its exponentials are done and
// the MMA thread issues that chunk's share of PV_X at once, so PV_X overlaps
// the rest of the softmax instead of following it.
// Per tile, kPChunks barrier slots; a kernel uses PChunks<...>::kCount of them.
// (The slot count is kept at the largest kCount: the barrier block and the
// shared-memory layout after it then match the one-chunk kernel's.)
// Calibration with O (whose softmax still has the mass partials to add after
// P is stored) gains from 2 chunks of 64 keys, each signalled per warp
// (967 vs 947 TFLOP/s in an interleaved same-box A/B; 4 chunks: 900); pruned
// attention and S-CAS-only calibration measured best with one P store
// signalled by every thread (2-7% and 6% ahead of 2 chunks).
constexpr int kPChunks = 2;
template <bool MASS, bool WITH_O>
struct PChunks {
  static constexpr int kCount = (MASS && WITH_O) ? 2 : 1;
  static constexpr int kKeys = kBlockN / kCount;          // keys per chunk
  static constexpr bool kPerWarp = kCount > 1;             // one arrival per warp (else per thread)
  static constexpr int kArrivals = kPerWarp ? kBlockM / 32 : kBlockM;
};

enum Bar {
  kBarQ = 0,
  kBarKFull = 1,      // [2]
  kBarVFull = 3,      // [2]
  kBarKEmpty = 5,     // [2]
  kBarVEmpty = 7,     // [2]
  kBarSFull = 9,      // [tile]
  kBarPFull = 11,     // [tile][kPChunks]; without O, chunk 0 = "S_X read"
  kBarODone = 15,     // [tile]
  kBarDrain = 17,
  kNumBars = 18
};

// Store one P chunk (kKeys / 2 columns of bf16 pairs) into TMEM.
VARK_DEV void tmem_st_chunk(uint32_t taddr, const uint32_t (&r)[32]) { tmem_st32(taddr, r); }
VARK_DEV void tmem_st_chunk(uint32_t taddr, const uint32_t (&r)[64]) {
  tmem_st32(taddr, reinterpret_cast<const uint32_t(&)[32]>(r[0]));
  tmem_st32(taddr + 32, reinterpret_cast<const uint32_t(&)[32]>(r[32]));
}

// Dynamic shared memory a CTA may opt into on sm_100 (227 KB).
constexpr int kMaxSmemOptin = 232448;

// Shared-memory layout.  QB = 0: bf16 K/V by TMA.  QB = 8, 4, 3 (pruned
// attention over a packed past): after the per-CTA tables, the converter's
// barriers and kCodeSlots staging slots, each holding one K or V tile's codes.
template <int D, int QB = 0>
struct Smem {
  static constexpr int kQPanels = D / 64;
  static constexpr int kTile = kQPanels * kPanelBytes;
  static constexpr int kQ = 0;                          // [2 tiles]
  static constexpr int kK = kQ + 2 * kTile;             // [2 stages]
  static constexpr int kV = kK + kStages * kTile;       // [2 stages]
  static constexpr int kBar = kV + kStages * kTile;
  static constexpr int kMisc = kBar + kNumBars * 8;     // tmem base, abort flag
  static constexpr int kRed = kMisc + 16;               // [2 tiles][4 warps][32] fp32
  static constexpr int kDesc = kRed + 2 * 4 * 32 * 4;   // [kMaxDesc] uint32 key-tile descriptors
  static constexpr int kBias2 = kDesc + kMaxDesc * 4;   // [32] fp32 bias * log2(e) of this head
  static constexpr int kSegOff = kBias2 + 32 * 4;       // [32] int32 this head's seg_off (pruned)
  static constexpr int kColBias = kSegOff + 32 * 4;     // [2 tiles][128] fp32 per-column bias / mask
  static constexpr int kMass = kColBias + 2 * 128 * 4;  // [2 tiles][S][128] fp32 (calibration)
  // packed past only (no mass there)
  static constexpr int kQBar = kMass;                   // [4] converter barriers
  static constexpr int kCode = kQBar + 128;             // [kCodeSlots] code tiles
  static constexpr int kCodeRowBytes = D * QB / 8;
  static constexpr int kSlotBytes = kBlockN * kCodeRowBytes;
  // two slots where they fit (16 bytes of over-read room for the 3-bit
  // groups of the last row, 1024 for the base alignment)
  static constexpr int kCodeSlots = (kCode + 2 * kSlotBytes + 16 + 1024 <= kMaxSmemOptin) ? 2 : 1;
  static int alloc(bool mass, int S) {
    if (QB != 0) return kCode + kCodeSlots * kSlotBytes + 16 + 1024;
    return kMass + (mass ? 2 * S * kBlockM * 4 : 0) + 1024;
  }
};

// Tile j of the key list of one work item.
struct KTile {
  int src;        // 0: dense K/V ([B*H][T][D] map), 1: compacted K/V ([rows][D] map)
  int row;        // first row (dense: within (b,h); compacted: absolute)
  int valid;      // valid key columns in this tile
  int key0;       // first key index in the item's key list (segment coordinates)
};

template <bool PRUNED>
struct Item {
  int b, h, bh, k, row0;
  int rows_valid[2];
  int n_tiles;
  int n_past;      // PRUNED: tiles over the compacted past
  int past;        // PRUNED: past_len[h][k]
  int64_t kc_row0; // PRUNED: first compacted row of (b, h)

  __device__ KTile tile(const Params& p, int j) const {
    KTile t;
    if (!PRUNED) {
      const int Lk = p.sc.off[k] + p.sc.n[k];
      t.src = 0;
      t.row = j * kBlockN;
      t.valid = min(kBlockN, Lk - t.row);
      t.key0 = t.row;
    } else if (j < n_past) {
      t.src = 1;
      t.row = int(kc_row0 + int64_t(j) * kBlockN);
      t.valid = min(kBlockN, past - j * kBlockN);
      t.key0 = j * kBlockN;
    } else {
      const int jj = j - n_past;
      t.src = 0;
      t.row = (p.local_scale_only ? 0 : p.sc.off[k]) + jj * kBlockN;
      t.valid = min(kBlockN, p.sc.n[k] - jj * kBlockN);
      t.key0 = jj * kBlockN;
    }
    return t;
  }
};

template <bool PRUNED>
__device__ Item<PRUNED> decode_item(const Params& p) {
  Item<PRUNED> it;
  // Groups of G (batch, head) blocks, one after another: the CTAs in
  // flight share a few heads' K/V in L2.  Inside a group the order is pair-
  // major (heaviest pair of every head of the group first), so each launch
  // ends on light CTAs instead of a last head's heaviest ones.
  const int BH = p.B * p.H;
  constexpr int G = HeadGroup<PRUNED>::value;
  const int per_group = G * p.n_pairs;
  const int grp = blockIdx.x / per_group;
  const int g0 = grp * G;
  const int gsize = min(G, BH - g0);
  const int within = blockIdx.x - grp * per_group;
  it.bh = g0 + within % gsize;
  const int pi = within / gsize;
  it.b = it.bh / p.H;
  it.h = it.bh % p.H;
  const uint32_t e = p.pair[pi];
  it.k = int(e >> 24);
  it.row0 = int(e & 0xFFFFFFu);
  const int nk = p.sc.n[it.k];
  it.rows_valid[0] = min(kBlockM, nk - it.row0);
  it.rows_valid[1] = max(0, min(kBlockM, nk - it.row0 - kBlockM));
  if (!PRUNED) {
    const int Lk = p.sc.off[it.k] + nk;
    it.n_tiles = (Lk + kBlockN - 1) / kBlockN;
    it.n_past = 0;
    it.past = 0;
    it.kc_row0 = 0;
  } else {
    it.past = p.past_len[it.h * p.sc.S + it.k];
    it.n_past = (it.past + kBlockN - 1) / kBlockN;
    it.n_tiles = it.n_past + (nk + kBlockN - 1) / kBlockN;
    it.kc_row0 = int64_t(it.b) * p.R_l + p.head_off[it.h];
  }
  return it;
}

// Calls f(col_begin, col_end, scale) for every source-scale segment of the
// valid columns of a key tile, in column order.  segoff: this head's seg_off
// row (pruned attention).
template <bool PRUNED, typename F>
__device__ __forceinline__ void for_each_segment(const Params& p, const Item<PRUNED>& it, const KTile& t,
                                                 const int32_t* segoff, F&& f) {
  if (!PRUNED) {
    const int lo = t.key0, hi = t.key0 + t.valid;
    for (int s = 0; s <= it.k; ++s) {
      const int a = max(p.sc.off[s], lo), e = min(p.sc.off[s] + p.sc.n[s], hi);
      if (a < e) f(a - lo, e - lo, s);
    }
  } else if (t.src == 1) {
    const int lo = t.key0, hi = t.key0 + t.valid;
    for (int s = 0; s < it.k; ++s) {
      const int so = segoff[s];
      if (so < 0) continue;
      const int a = max(so, lo), e = min(so + p.sc.n[s], hi);
      if (a < e) f(a - lo, e - lo, s);
    }
  } else {
    f(0, t.valid, it.k);
  }
}

// Key-tile descriptor: bit 0 = one source scale and all 128 columns valid;
// bits 8..15 = the scale of the first column; bits 16..31 = valid columns.
template <bool PRUNED>
__device__ __forceinline__ uint32_t make_desc(const Params& p, const Item<PRUNED>& it, int j,
                                              const int32_t* segoff) {
  const KTile t = it.tile(p, j);
  int nseg = 0, sc = -1;
  for_each_segment<PRUNED>(p, it, t, segoff, [&](int, int, int s) {
    ++nseg;
    if (sc < 0) sc = s;
  });
  return uint32_t(nseg == 1 && t.valid == kBlockN) | (uint32_t(max(sc, 0)) << 8) | (uint32_t(t.valid) << 16);
}

// Source scale of column c of a key tile (c < valid); s0 = the scale of the
// tile's first column.
template <bool PRUNED>
__device__ __forceinline__ int column_scale(const Params& p, const Item<PRUNED>& it, const KTile& t, int c,
                                            const int32_t* segoff, int s0) {
  const int key = t.key0 + c;
  if (!PRUNED) {
    int s = s0;
    while (s < it.k && key >= p.sc.off[s + 1]) ++s;
    return s;
  } else if (t.src == 1) {
    int sc = s0;
    for (int s = s0; s < it.k; ++s) {
      const int so = segoff[s];
      if (so >= 0 && key >= so && key < so + p.sc.n[s]) sc = s;
    }
    return sc;
  }
  return it.k;
}

// ------------------------------------------------------------ packed past
// Pruned attention over a quantised retained cache (QB = 8, 4 or 3 bits per
// element in per-(block, channel) groups, as on the VAR-Q summary page, Key
// Contributions): warps 2 and 3 of the control warpgroup, idle in the bf16
// kernel, fill the K and V stages of every past tile themselves.  For each K
// or V tile one thread bulk-copies the tile's packed rows (contiguous in the
// compacted layout) into a staging slot; the 64 threads then expand every
// 8-channel group to bf16(code * scale) -- the product in fp32, the same
// arithmetic as the separate dequantiser, so the tile equals the dequantised
// cache bit for bit -- and store it in the 128-byte-swizzled layout a TMA
// load produces.  Rows past the tile's keys are zeros (their columns are
// masked, and zero V rows keep P * V finite).  Local-scale tiles still come by
// TMA from the producer.
//
// Barrier protocol.  Each stage's "empty" barrier is waited on by the
// converters for past tiles and by the producer for local tiles, and its
// "full" barrier gets one arrival per tile from whichever role fills it.  A
// parity wait is exact only while the waiter is at most one phase behind, so
// the producer, which skips the past tiles, makes its first stage wait only
// after the converters have passed all of theirs (kQBarConvDone); from then
// on the phase it waits for is the current one or the last completed one.
constexpr int kConvThreads = 64;
constexpr int kConvBar = 5;          // named barrier of the converter warps
constexpr int kQBarConvDone = 0;     // the converters are past their last stage wait
constexpr int kQBarCode = 1;         // [kCodeSlots] a slot's codes have landed

// Eight channels' codes -> four bf16 pairs (channels (0,1) .. (6,7)).  A
// code's biased value placed in the low mantissa bits of 1.5 * 2^23 reads
// 1.5 * 2^23 + biased, so one exact subtraction leaves the code; the product
// with the fp32 scale is rounded to fp32 (exact below 8 bits) and then to bf16.
// 4-bit codes take packed bf16 arithmetic instead: a nibble pair masked into
// bf16 pairs 128 + n (exponent 2^7, the nibble as the low mantissa bits),
// minus 136 leaves the codes exactly, and one bf16x2 multiply by the table's
// scale pair rounds the exact product once -- the same value as the fp32 path.
VARK_DEV uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
VARK_DEV uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
VARK_DEV uint4 expand_codes4(uint32_t w, const uint32_t (&sp)[4]) {
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t biased = ((w >> (4 * i)) & 0x000F000Fu) | 0x43004300u;   // channel 2i low, 2i + 1 high
    o[i] = bf16x2_mul(bf16x2_sub(biased, 0x43084308u), sp[i]);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}
template <int QB>
VARK_DEV uint4 expand_codes(uint32_t w0, uint32_t w1, const float (&sc)[8]) {
  constexpr float kBias = 12582912.0f + (QB == 8 ? 128.f : QB == 4 ? 8.f : 4.f);
  uint32_t u[8];
  if constexpr (QB == 8) {          // bytes 0-3 of w0, then of w1; sign flipped: code + 128
    const uint32_t a = w0 ^ 0x80808080u, b = w1 ^ 0x80808080u;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      u[i] = __byte_perm(a, 0x4B400000u, 0x7640u | uint32_t(i));
      u[4 + i] = __byte_perm(b, 0x4B400000u, 0x7640u | uint32_t(i));
    }
  } else if constexpr (QB == 4) {   // channel 2i at bit 4i, 2i + 1 at bit 16 + 4i: code + 8
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      u[2 * i] = 0x4B400000u | ((w0 >> (4 * i)) & 0xFu);
      u[2 * i + 1] = 0x4B400000u | ((w0 >> (16 + 4 * i)) & 0xFu);
    }
  } else {                          // channel i at bit 3i of a 24-bit group: code + 4
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = 0x4B400000u | ((w0 >> (3 * i)) & 0x7u);
  }
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float c0, c1, v0, v1;
    fadd2(c0, c1, __uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]), -kBias, -kBias);
    // + (-0): the plain product, signed zeros included
    ffma2(v0, v1, c0, c1, sc[2 * i], sc[2 * i + 1], -0.f, -0.f);
    o[i] = pack_bf16x2(v0, v1);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// The 8 channel scales of one (batch, head, scale) table row from channel
// 8 * group on: 8-bit tables hold the fp32 absmax a (scale a / 127, IEEE
// division), 4- and 3-bit tables the bf16 scale bits (4-bit: kept as the
// table's channel pairs, sc unused).
VARK_DEV void load_scale_pairs(const void* tab, int64_t idx, uint32_t (&sp)[4]) {
  const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(tab) + idx));
  sp[0] = w.x; sp[1] = w.y; sp[2] = w.z; sp[3] = w.w;
}
template <int QB>
VARK_DEV void load_scales(const void* tab, int64_t idx, float (&sc)[8]) {
  if constexpr (QB == 8) {
    const float4* a = reinterpret_cast<const float4*>(static_cast<const float*>(tab) + idx);
    const float4 x = __ldg(a), y = __ldg(a + 1);
    sc[0] = x.x / 127.f; sc[1] = x.y / 127.f; sc[2] = x.z / 127.f; sc[3] = x.w / 127.f;
    sc[4] = y.x / 127.f; sc[5] = y.y / 127.f; sc[6] = y.z / 127.f; sc[7] = y.w / 127.f;
  } else {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(tab) + idx));
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      sc[2 * e] = __uint_as_float(ws[e] << 16);
      sc[2 * e + 1] = __uint_as_float(ws[e] & 0xFFFF0000u);
    }
  }
}

// One K or V past tile from its staged codes into a stage.  Thread ct owns the
// 8-channel group ct % (D / 8) of every (kConvThreads / (D / 8))-th row; a
// row's scales are those of the kept scale whose segment holds its key.  Rows
// go kRowsInFlight at a time: their code loads first, then the expansions.
template <int D, int QB>
VARK_DEV void expand_tile(const Params& p, const Item<true>& it, const KTile& t, const void* tab, uint32_t slot,
                          uint32_t stage, int ct) {
  using L = Smem<D, QB>;
  constexpr int kGroups = D / 8;
  constexpr int kRowStep = kConvThreads / kGroups;
  constexpr int kRowsInFlight = QB == 4 ? 4 : 2;
  static_assert((kBlockN / kRowStep) % kRowsInFlight == 0, "rows per thread");
  const int cw = ct % kGroups;
  const uint32_t dst = stage + uint32_t(cw >> 3) * kPanelBytes;   // the group's 64-channel panel
  const uint32_t chunk = uint32_t(cw & 7);                          // its 16-byte chunk in a row
  const int S = p.sc.S;
  const int32_t* segoff = p.seg_off + it.h * S;
  const int64_t tab0 = (int64_t(it.b) * p.H + it.h) * S * D + cw * 8;
  int s = -1, seg_hi = -1;   // the kept segment [.., seg_hi) of the current key
  float sc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  uint32_t sp[4] = {0u, 0u, 0u, 0u};
#pragma unroll 1
  for (int r0 = ct / kGroups; r0 < kBlockN; r0 += kRowsInFlight * kRowStep) {
    uint32_t w0[kRowsInFlight], w1[kRowsInFlight];
#pragma unroll
    for (int i = 0; i < kRowsInFlight; ++i) {
      const int r = r0 + i * kRowStep;
      const uint32_t at = slot + uint32_t(r * L::kCodeRowBytes + cw * QB);
      w0[i] = w1[i] = 0u;
      if (r < t.valid) {
        if constexpr (QB == 8) {
          w0[i] = ld_shared_u32(at);
          w1[i] = ld_shared_u32(at + 4);
        } else if constexpr (QB == 4) {
          w0[i] = ld_shared_u32(at);
        } else {   // a 24-bit group at any byte offset: two aligned words, funnel-shifted
          w0[i] = __funnelshift_r(ld_shared_u32(at & ~3u), ld_shared_u32((at & ~3u) + 4u), (at & 3u) * 8u);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kRowsInFlight; ++i) {
      const int r = r0 + i * kRowStep;
      uint4 o = make_uint4(0u, 0u, 0u, 0u);   // rows past the tile's keys: zeros
      if (r < t.valid) {
        const int key = t.key0 + r;
        if (key >= seg_hi) {
          do {
            ++s;
          } while (s < it.k && (__ldg(segoff + s) < 0 || key >= __ldg(segoff + s) + p.sc.n[s]));
          seg_hi = __ldg(segoff + s) + p.sc.n[s];
          if constexpr (QB == 4) load_scale_pairs(tab, tab0 + int64_t(s) * D, sp);
          else load_scales<QB>(tab, tab0 + int64_t(s) * D, sc);
        }
        if constexpr (QB == 4) o = expand_codes4(w0[i], sp);
        else o = expand_codes<QB>(w0[i], w1[i], sc);
      }
      st_shared_v4(dst + uint32_t(r) * 128u + ((chunk ^ uint32_t(r & 7)) << 4), o);
    }
  }
}

// The converter role: K then V of past tiles 0 .. n_past - 1, in order.
template <int D, int QB>
VARK_DEV void convert_past(const Params& p, const Item<true>& it, uint32_t sK, uint32_t sV, uint32_t sCode,
                           uint32_t bar0, uint32_t qbar0, volatile int* abort_flag, int ct) {
  using L = Smem<D, QB>;
  constexpr int kSlots = L::kCodeSlots;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  auto qbar = [&](int i) { return qbar0 + 8u * uint32_t(i); };
  const int n_conv = p.withhold_tile < 0 ? it.n_past : min(it.n_past, p.withhold_tile);
  const int U = 2 * n_conv;   // unit u: tile u / 2, K (u even) or V (u odd)
  // (thread 0) copy of unit u's packed rows into slot u % kSlots
  auto issue = [&](int u) -> bool {
    const KTile t = it.tile(p, u >> 1);
    if (t.row < 0 || int64_t(t.row) + t.valid > p.kc_rows) {   // tables inconsistent with the cache size
      atomicExch(p.status, VARK_E_SHAPE);
      *abort_flag = 1;
      return false;
    }
    const int sl = u % kSlots;
    const uint32_t bytes = uint32_t(t.valid) * uint32_t(L::kCodeRowBytes);
    const uint8_t* src = static_cast<const uint8_t*>((u & 1) ? p.vq : p.kq) + int64_t(t.row) * L::kCodeRowBytes;
    mbar_arrive_expect_tx(qbar(kQBarCode + sl), bytes);
    bulk_load(sCode + uint32_t(sl * L::kSlotBytes), src, bytes, qbar(kQBarCode + sl));
    return true;
  };
  int issued = 0;        // thread 0: units whose copy is issued
  bool copy_ok = true;
  if (ct == 0)
    while (copy_ok && issued < min(U, kSlots)) {
      copy_ok = issue(issued);
      if (copy_ok) ++issued;
    }
  int u = 0;
  for (; u < U; ++u) {
    const int j = u >> 1, which = u & 1, st = j % kStages;
    // the stage is free once the MMAs of tile j - kStages have read it
    bool go = j < kStages || mbar_wait(bar((which ? kBarVEmpty : kBarKEmpty) + st), ((j / kStages) - 1) & 1,
                                       abort_flag, p.status, p.wait_limit_ns);
    if (!bar_and(kConvBar, kConvThreads, go)) break;
    if (u == U - 1 && ct == 0) mbar_arrive(qbar(kQBarConvDone));
    go = mbar_wait(qbar(kQBarCode + u % kSlots), (u / kSlots) & 1, abort_flag, p.status, p.wait_limit_ns);
    if (!bar_and(kConvBar, kConvThreads, go)) break;
    expand_tile<D, QB>(p, it, it.tile(p, j), which ? p.vtab : p.ktab, sCode + uint32_t((u % kSlots) * L::kSlotBytes),
                       (which ? sV : sK) + uint32_t(st * L::kTile), ct);
    fence_proxy_async_smem();                  // the stage's stores, before the tensor core reads them
    named_bar_sync(kConvBar, kConvThreads);     // the stage is written and the slot read by all
    if (ct == 0) {
      mbar_arrive(bar((which ? kBarVFull : kBarKFull) + st));
      if (copy_ok && issued < U) {
        fence_proxy_async_smem();              // the slot's reads, before the copy overwrites it
        copy_ok = issue(issued);
        if (copy_ok) ++issued;
      }
    }
  }
  // Drain (abort path): copies still in flight land before the CTA exits.
  if (ct == 0) {
    volatile int no_abort = 0;
    for (int v = u; v < issued; ++v) mbar_wait(qbar(kQBarCode + v % kSlots), (v / kSlots) & 1, &no_abort, nullptr);
  }
}

// WITH_O = false (calibration called without an output): no V tiles and no PV
// MMAs; the softmax releases S_X as soon as it has read it into registers, so
// the next S MMA of that tile overlaps the rest of its softmax.
// QB != 0: pruned attention whose past comes as packed codes (converter warps).
template <int D, bool PRUNED, bool MASS, bool WITH_O, int QB = 0>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
            const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ Params p) {
  static_assert(QB == 0 || (PRUNED && WITH_O && !MASS), "packed past: pruned attention only");
  using L = Smem<D, QB>;
  using PC = PChunks<MASS, WITH_O>;
  constexpr int QP = L::kQPanels;
  constexpr uint32_t kTileBytes = L::kTile;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the shared array itself so the
  // compiler keeps shared-space loads and stores
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::kQ, sK = sbase + L::kK, sV = sbase + L::kV;
  float* red_sm = reinterpret_cast<float*>(smem + L::kRed);
  float* mass_sm = reinterpret_cast<float*>(smem + L::kMass);
  const uint32_t bar0 = sbase + L::kBar;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Item<PRUNED> it = decode_item<PRUNED>(p);
  const int n = it.n_tiles;
  const int n_act = it.rows_valid[1] > 0 ? 2 : 1;   // active query tiles

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bar(kBarSFull + x), 1);
      for (int c = 0; c < kPChunks; ++c) mbar_init(bar(kBarPFull + x * kPChunks + c), PC::kArrivals);
      mbar_init(bar(kBarODone + x), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    if constexpr (QB != 0) {
      mbar_init(sbase + L::kQBar + 8u * kQBarConvDone, 1);
      for (int sl = 0; sl < L::kCodeSlots; ++sl) mbar_init(sbase + L::kQBar + 8u * (kQBarCode + sl), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
    // Start the first loads now, so their latency overlaps TMEM allocation
    // and the table setup below (the producer loop continues after them).
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (PRUNED) {
      tma_prefetch_desc(&tm_kc);
      tma_prefetch_desc(&tm_vc);
    }
    const int qrow = (p.q_scale_rows ? 0 : p.sc.off[it.k]) + it.row0;
    mbar_arrive_expect_tx(bar(kBarQ), n_act * kTileBytes);
    for (int x = 0; x < n_act; ++x)
      for (int c = 0; c < QP; ++c)
        tma_load_3d(sQ + x * kTileBytes + c * kPanelBytes, &tm_q, bar(kBarQ), c * 64, qrow + x * kBlockM, it.bh);
    const int first = min(min(n, kStages), p.withhold_tile < 0 ? n : p.withhold_tile);
    for (int j = 0; j < first; ++j) {
      const KTile t = it.tile(p, j);
      if (QB != 0 && t.src == 1) continue;   // a past tile: the converters fill it
      mbar_arrive_expect_tx(bar(kBarKFull + j), kTileBytes);
      for (int c = 0; c < QP; ++c) {
        const uint32_t dst = sK + j * kTileBytes + c * kPanelBytes;
        if (t.src == 0) tma_load_3d(dst, &tm_k, bar(kBarKFull + j), c * 64, t.row, it.bh);
        else tma_load_2d(dst, &tm_kc, bar(kBarKFull + j), c * 64, t.row);
      }
      if (!WITH_O) continue;
      mbar_arrive_expect_tx(bar(kBarVFull + j), kTileBytes);
      for (int c = 0; c < QP; ++c) {
        const uint32_t dst = sV + j * kTileBytes + c * kPanelBytes;
        if (t.src == 0) tma_load_3d(dst, &tm_v, bar(kBarVFull + j), c * 64, t.row, it.bh);
        else tma_load_2d(dst, &tm_vc, bar(kBarVFull + j), c * 64, t.row);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    setmaxnreg_dec56();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- producer
      // (Q and the first kStages key tiles were issued right after the
      // barrier initialisation, by this same thread.)
      int issued_k = min(min(n, kStages), p.withhold_tile < 0 ? n : p.withhold_tile);
      int issued_v = WITH_O ? issued_k : 0;
      bool conv_passed = QB == 0 || it.n_past == 0;   // packed past: the converters' stage waits are behind
      for (int j = issued_k; j < n; ++j) {
        const int st = j % kStages;
        const KTile t = it.tile(p, j);
        if (j == p.withhold_tile) break;   // test hook: this tile never arrives
        if (QB != 0 && t.src == 1) continue;   // a past tile: the converters fill it
        if (j >= kStages && !conv_passed) {
          if (!mbar_wait(sbase + L::kQBar + 8u * kQBarConvDone, 0, abort_flag, p.status, p.wait_limit_ns)) break;
          conv_passed = true;
        }
        if (j >= kStages && !mbar_wait(bar(kBarKEmpty + st), ((j / kStages) - 1) & 1, abort_flag, p.status, p.wait_limit_ns)) break;
        mbar_arrive_expect_tx(bar(kBarKFull + st), kTileBytes);
        for (int c = 0; c < QP; ++c) {
          const uint32_t dst = sK + st * kTileBytes + c * kPanelBytes;
          if (t.src == 0) tma_load_3d(dst, &tm_k, bar(kBarKFull + st), c * 64, t.row, it.bh);
          else tma_load_2d(dst, &tm_kc, bar(kBarKFull + st), c * 64, t.row);
        }
        issued_k = j + 1;
        if (!WITH_O) continue;
        if (j >= kStages && !mbar_wait(bar(kBarVEmpty + st), ((j / kStages) - 1) & 1, abort_flag, p.status, p.wait_limit_ns)) break;
        mbar_arrive_expect_tx(bar(kBarVFull + st), kTileBytes);
        for (int c = 0; c < QP; ++c) {
          const uint32_t dst = sV + st * kTileBytes + c * kPanelBytes;
          if (t.src == 0) tma_load_3d(dst, &tm_v, bar(kBarVFull + st), c * 64, t.row, it.bh);
          else tma_load_2d(dst, &tm_vc, bar(kBarVFull + st), c * 64, t.row);
        }
        issued_v = j + 1;
      }
      // Drain: every load issued here has landed before the CTA exits
      // (immediate on the normal path; bounded on the abort path).
      // (Past tiles of a packed past are the converters'; they have no copy.)
      volatile int no_abort = 0;
      const int own0 = QB != 0 ? it.n_past : 0;
      mbar_wait(bar(kBarQ), 0, &no_abort, nullptr);
      for (int j = max(own0, issued_k - kStages); j < issued_k; ++j)
        mbar_wait(bar(kBarKFull + j % kStages), (j / kStages) & 1, &no_abort, nullptr);
      for (int j = max(own0, issued_v - kStages); j < issued_v; ++j)
        mbar_wait(bar(kBarVFull + j % kStages), (j / kStages) & 1, &no_abort, nullptr);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, false, true);
      auto issue_s = [&](int x, int st) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
          const uint64_t a = smem_desc_sw128(sQ + x * kTileBytes + off, 16, 1024);
          const uint64_t b = smem_desc_sw128(sK + st * kTileBytes + off, 16, 1024);
          mma_bf16_ss(tmem + x * kBlockN, a, b, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // PV_X of key tile jp from the V stage pst, one P chunk at a time: each
      // chunk's two K = 16 steps are issued as soon as the softmax has stored
      // that chunk.  Returns false on abort.
      auto issue_pv = [&](int x, int pst, int jp) -> bool {
#pragma unroll
        for (int c = 0; c < PC::kCount; ++c) {
          if (!mbar_wait(bar(kBarPFull + x * kPChunks + c), jp & 1, abort_flag, p.status, p.wait_limit_ns))
            return false;
          tc_fence_after();
#pragma unroll
          for (int kq = 0; kq < PC::kKeys / 16; ++kq) {
            const int kk = c * (PC::kKeys / 16) + kq;
            const uint64_t b = smem_desc_sw128(sV + pst * kTileBytes + kk * 2048, kPanelBytes, 1024);
            mma_bf16_ts(tmem + 256 + x * D, tmem + x * kBlockN + kk * 8, b, idesc_o, (jp > 0 || kk > 0) ? 1u : 0u);
          }
        }
        return true;
      };
      bool ok = mbar_wait(bar(kBarQ), 0, abort_flag, p.status, p.wait_limit_ns);
      if (!WITH_O) {
        // S MMAs only: S_X(j) once the softmax has read S_X(j-1)
        for (int j = 0; ok && j < n; ++j) {
          const int st = j % kStages;
          if (!(ok = mbar_wait(bar(kBarKFull + st), (j / kStages) & 1, abort_flag, p.status, p.wait_limit_ns))) break;
          for (int x = 0; x < n_act; ++x) {
            if (j > 0 && !(ok = mbar_wait(bar(kBarPFull + x * kPChunks), (j - 1) & 1, abort_flag, p.status, p.wait_limit_ns))) break;
            tc_fence_after();
            issue_s(x, st);
            mma_commit(bar(kBarSFull + x));
          }
          if (!ok) break;
          if (j + kStages < n) mma_commit(bar(kBarKEmpty + st));
        }
      }
      for (int j = 0; WITH_O && ok && j < n; ++j) {
        const int st = j % kStages, pst = (j + kStages - 1) % kStages;
        if (!(ok = mbar_wait(bar(kBarKFull + st), (j / kStages) & 1, abort_flag, p.status, p.wait_limit_ns))) break;
        if (j > 0 && !(ok = mbar_wait(bar(kBarVFull + pst), ((j - 1) / kStages) & 1, abort_flag, p.status, p.wait_limit_ns))) break;
        for (int x = 0; x < n_act; ++x) {
          if (j > 0) {
            if (!(ok = issue_pv(x, pst, j - 1))) break;
          } else {
            tc_fence_after();
          }
          issue_s(x, st);
          mma_commit(bar(kBarSFull + x));
        }
        if (!ok) break;
        if (j + kStages < n) mma_commit(bar(kBarKEmpty + st));
        if (j > 0 && (j - 1) + kStages < n) mma_commit(bar(kBarVEmpty + pst));
      }
      if (WITH_O && ok && n > 0) {
        const int pst = (n - 1) % kStages;
        ok = mbar_wait(bar(kBarVFull + pst), ((n - 1) / kStages) & 1, abort_flag, p.status, p.wait_limit_ns);
        for (int x = 0; ok && x < n_act; ++x) {
          if (!(ok = issue_pv(x, pst, n - 1))) break;
          mma_commit(bar(kBarODone + x));
        }
      }
      // Drain: all MMAs of this thread complete before TMEM is released.
      mma_commit(bar(kBarDrain));
      volatile int no_abort = 0;
      mbar_wait(bar(kBarDrain), 0, &no_abort, nullptr);
    } else if (QB != 0 && (warp == 2 || warp == 3)) {
      // ---------------------------------------------------------- packed-past converters
      if constexpr (QB != 0)
        convert_past<D, QB>(p, it, sK, sV, sbase + L::kCode, bar0, sbase + L::kQBar, abort_flag, threadIdx.x - 64);
    }
  } else {
    setmaxnreg_inc224();
    // ------------------------------------------------------------ softmax
    const int x = (warp >> 2) - 1;                    // query tile 0 (A) or 1 (B)
    const int r = threadIdx.x - 128 * (x + 1);        // row within the tile = TMEM lane
    const int t256 = threadIdx.x - 128;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + x * kBlockN + lane_base;
    const uint32_t tO = tmem + 256 + x * D + lane_base;
    const bool active = x < n_act;
    const float qk2 = p.tau[it.h] * p.scale_log2;
    uint32_t* desc_sm = reinterpret_cast<uint32_t*>(smem + L::kDesc);
    float* bias2_sm = reinterpret_cast<float*>(smem + L::kBias2);
    int32_t* segoff_sm = reinterpret_cast<int32_t*>(smem + L::kSegOff);
    float* colbias = reinterpret_cast<float*>(smem + L::kColBias) + x * kBlockN;
    float* mrow = mass_sm + (x * p.sc.S) * kBlockM + r;   // [s] stride kBlockM

    // Per-CTA tables, shared by both tiles: bias * log2(e) per source scale,
    // this head's seg_off row, and the descriptor of every key tile.
    if (t256 < p.sc.S) {
      bias2_sm[t256] = p.bias ? p.bias[it.h * p.sc.S + t256] * kLog2e : 0.f;
      if (PRUNED) segoff_sm[t256] = p.seg_off[it.h * p.sc.S + t256];
    }
    named_bar_sync(2, 2 * kBlockM);
    for (int jj = t256; jj < min(n, kMaxDesc); jj += 2 * kBlockM) desc_sm[jj] = make_desc<PRUNED>(p, it, jj, segoff_sm);
    named_bar_sync(2, 2 * kBlockM);

    float m_used = -INFINITY, l_sum = 0.f;
    if (MASS)
      for (int s = 0; s < p.sc.S; ++s) mrow[s * kBlockM] = 0.f;
    bool ok = active;

    for (int j = 0; ok && j < n; ++j) {
      const uint32_t d = j < kMaxDesc ? desc_sm[j] : make_desc<PRUNED>(p, it, j, segoff_sm);
      const bool fast = (d & 1u) && (qk2 > 0.f);
      const int seg_scale = int((d >> 8) & 0xFFu);
      // the tile's 128 threads agree on continuing (a per-column table and a
      // named barrier may follow)
      ok = bar_and(3 + x, kBlockM, mbar_wait(bar(kBarSFull + x), j & 1, abort_flag, p.status, p.wait_limit_ns));
      if (!ok) break;
      tc_fence_after();
      float sv[kBlockN];
      {
        uint32_t v[kBlockN / 32][32];
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) tmem_ld32(tS + c * 32, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) {
          reg_fence32(v[c]);
#pragma unroll
          for (int i = 0; i < 32; ++i) sv[c * 32 + i] = __uint_as_float(v[c][i]);
        }
      }
      if (!WITH_O) {   // S_X is in registers: the next S MMA of this tile may overwrite it
        tc_fence_before();
        mbar_arrive(bar(kBarPFull + x * kPChunks));
      }
      // Exponent of column c: sv[c] * qk2 + (b2 - m) on a full single-scale
      // tile (fast), sv[c] * qk2 + colbias[c] - m otherwise.  In calibration
      // with O, after the first tile, a fast tile's first kSpecKeys columns are
      // exponentiated against the running max while the tile's row max is
      // taken alongside, so the max is off the S -> P -> PV -> S chain; a row
      // whose max grew by more than the threshold (rare after the first
      // tiles) rescales and recomputes those columns from S_X, which is still
      // in TMEM.  (Measured +4.5% on calibration, -2% on pruned attention,
      // which therefore takes the max first.)
      constexpr int kPoly = WITH_O ? kPolyPer8 : kPolyPer8NoO;
      auto exp_fast = [&](float* cv, float shift, auto ncols) {
        constexpr int kN = decltype(ncols)::value;
#pragma unroll
        for (int c = 0; c < kN; c += 2) ffma2(cv[c], cv[c + 1], cv[c], cv[c + 1], qk2, qk2, shift, shift);
#pragma unroll
        for (int c = 0; c < kN; c += 8) {
#pragma unroll
          for (int i = 0; i < kPoly; i += 2) exp2_poly2(cv[c + i], cv[c + i + 1]);
#pragma unroll
          for (int i = kPoly; i < 8; ++i) cv[c + i] = ex2_approx(cv[c + i]);
        }
      };
      const bool spec = MASS && WITH_O && fast && j > 0;
      float b2 = 0.f, m_tile;
      if (fast) {
        // one source scale, all columns valid
        b2 = bias2_sm[seg_scale];
        float m0 = sv[0], m1 = sv[1], m2 = sv[2], m3 = sv[3];
#pragma unroll
        for (int c = 4; c < kBlockN - 4; c += 8) {
          m0 = fmax3(m0, sv[c + 0], sv[c + 1]);
          m1 = fmax3(m1, sv[c + 2], sv[c + 3]);
          m2 = fmax3(m2, sv[c + 4], sv[c + 5]);
          m3 = fmax3(m3, sv[c + 6], sv[c + 7]);
        }
        m0 = fmax3(m0, sv[kBlockN - 4], sv[kBlockN - 3]);
        m1 = fmax3(m1, sv[kBlockN - 2], sv[kBlockN - 1]);
        if (spec) exp_fast(sv, b2 - m_used, Int<kSpecKeys>{});   // independent of the max above
        m_tile = fmaf(fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)), qk2, b2);
      } else {
        // boundary / tail tile: per-column bias (or -inf mask) from a table
        // the tile's 128 threads fill, one column each
        const KTile t = it.tile(p, j);
        colbias[r] = (r < t.valid) ? bias2_sm[column_scale<PRUNED>(p, it, t, r, segoff_sm, seg_scale)] : -INFINITY;
        named_bar_sync(3 + x, kBlockM);
#pragma unroll
        for (int c = 0; c < kBlockN; c += 4) {
          const float4 cb = *reinterpret_cast<const float4*>(colbias + c);
          ffma2(sv[c], sv[c + 1], sv[c], sv[c + 1], qk2, qk2, cb.x, cb.y);
          ffma2(sv[c + 2], sv[c + 3], sv[c + 2], sv[c + 3], qk2, qk2, cb.z, cb.w);
        }
        float m0 = sv[0], m1 = sv[1], m2 = sv[2], m3 = sv[3];
#pragma unroll
        for (int c = 4; c < kBlockN - 4; c += 8) {
          m0 = fmax3(m0, sv[c + 0], sv[c + 1]);
          m1 = fmax3(m1, sv[c + 2], sv[c + 3]);
          m2 = fmax3(m2, sv[c + 4], sv[c + 5]);
          m3 = fmax3(m3, sv[c + 6], sv[c + 7]);
        }
        m0 = fmax3(m0, sv[kBlockN - 4], sv[kBlockN - 3]);
        m1 = fmax3(m1, sv[kBlockN - 2], sv[kBlockN - 1]);
        m_tile = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
      }
      // Running max with a stale-max threshold; O_X is stable here (the
      // commit that completed S_X(j) also covers PV_X(j-1)).
      float f = 1.f;
      if (j == 0) {
        m_used = m_tile;
      } else if (m_tile > m_used + kRescaleThreshold) {
        f = ex2_approx(m_used - m_tile);
        m_used = m_tile;
        l_sum *= f;
        if (MASS)
          for (int s = 0; s <= it.k; ++s) mrow[s * kBlockM] *= f;
      }
      if (WITH_O && j > 0 && __any_sync(0xffffffffu, f != 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + c * 32, v);
          tmem_wait_ld();
          reg_fence32(v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
          tmem_st32(tO + c * 32, v);
        }
        if (spec) {
          // chunk 0 went against the old max in the rows that moved: reload
          // their scores and recompute
#pragma unroll
          for (int c = 0; c < kSpecKeys / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tS + c * 32, v);
            tmem_wait_ld();
            reg_fence32(v);
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[c * 32 + i] = (f != 1.f) ? __uint_as_float(v[i]) : sv[c * 32 + i];
          }
          if (f != 1.f) exp_fast(sv, b2 - m_used, Int<kSpecKeys>{});
        }
      }
      // p = 2^(exponent - m_used), one chunk of PC::kKeys columns at a time.
      // With O, chunk q's bf16 pairs go to TMEM (over S_X's first columns)
      // while chunk q+1's exponentials run, and the warp signals the chunk
      // to the MMA thread once its store has completed.
      const float shm = fast ? b2 - m_used : -m_used;
#pragma unroll
      for (int q = 0; q < PC::kCount; ++q) {
        float* cv = sv + q * PC::kKeys;
        if (fast) {
          if (!(spec && q == 0)) exp_fast(cv, shm, Int<PC::kKeys>{});
          else exp_fast(cv + kSpecKeys, shm, Int<PC::kKeys - kSpecKeys>{});
        } else {
#pragma unroll
          for (int c = 0; c < PC::kKeys; c += 2) fadd2(cv[c], cv[c + 1], cv[c], cv[c + 1], shm, shm);
#pragma unroll
          for (int c = 0; c < PC::kKeys; ++c) cv[c] = ex2_approx(cv[c]);
        }
        if (WITH_O) {
          if (q > 0) {   // chunk q-1's store has been in flight during these exponentials
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kBarPFull + x * kPChunks + q - 1));
          }
          uint32_t pk[PC::kKeys / 2];
#pragma unroll
          for (int c = 0; c < PC::kKeys / 2; ++c) pk[c] = pack_bf16x2(cv[2 * c], cv[2 * c + 1]);
          tmem_st_chunk(tS + q * (PC::kKeys / 2), pk);
        }
      }
      if (WITH_O) {
        tmem_wait_st();
        tc_fence_before();
        if (PC::kPerWarp) {
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(kBarPFull + x * kPChunks + PC::kCount - 1));
        } else {
          mbar_arrive(bar(kBarPFull + x * kPChunks + PC::kCount - 1));
        }
      }
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, a4 = 0.f, a5 = 0.f, a6 = 0.f, a7 = 0.f;
#pragma unroll
      for (int c = 0; c < kBlockN; c += 8) {
        fadd2(a0, a1, a0, a1, sv[c + 0], sv[c + 1]);
        fadd2(a2, a3, a2, a3, sv[c + 2], sv[c + 3]);
        fadd2(a4, a5, a4, a5, sv[c + 4], sv[c + 5]);
        fadd2(a6, a7, a6, a7, sv[c + 6], sv[c + 7]);
      }
      const float tile_sum = ((a0 + a1) + (a2 + a3)) + ((a4 + a5) + (a6 + a7));
      l_sum += tile_sum;
      if (MASS) {
        if (d & 1u) {
          mrow[seg_scale * kBlockM] += tile_sum;
        } else {
          // per source-scale segment: a 0/1 column weight table (one column
          // per thread) and a dot product with the row's probabilities
          const KTile t = it.tile(p, j);
          named_bar_sync(3 + x, kBlockM);   // every thread is done with colbias
          for_each_segment<PRUNED>(p, it, t, segoff_sm, [&](int cb, int ce, int s) {
            colbias[r] = (r >= cb && r < ce) ? 1.f : 0.f;
            named_bar_sync(3 + x, kBlockM);
            float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
            for (int c = 0; c < kBlockN; c += 4) {
              const float4 w4 = *reinterpret_cast<const float4*>(colbias + c);
              ffma2(acc0, acc1, sv[c], sv[c + 1], w4.x, w4.y, acc0, acc1);
              ffma2(acc2, acc3, sv[c + 2], sv[c + 3], w4.z, w4.w, acc2, acc3);
            }
            mrow[s * kBlockM] += (acc0 + acc1) + (acc2 + acc3);
            named_bar_sync(3 + x, kBlockM);
          });
        }
      }
    }

    // ---------------------------------------------------------- epilogue
    if (WITH_O && ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(kBarODone + x), 0, abort_flag, p.status, p.wait_limit_ns));
    const bool row_ok = ok && r < it.rows_valid[x];
    const float inv_l = 1.f / l_sum;
    if (WITH_O && ok && p.out != nullptr) {
      tc_fence_after();
      const int out_row = (p.q_scale_rows ? 0 : p.sc.off[it.k]) + it.row0 + x * kBlockM + r;
      uint16_t* orow = p.out + (int64_t(it.bh) * p.q_rows + out_row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        tmem_wait_ld();
        reg_fence32(v);
        if (row_ok) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * inv_l, __uint_as_float(v[8 * q + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * inv_l, __uint_as_float(v[8 * q + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * inv_l, __uint_as_float(v[8 * q + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * inv_l, __uint_as_float(v[8 * q + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + c * 32 + q * 8) = w;
          }
        }
      }
    }
    if (MASS) {
      // mean over the B * n_k rows of scale k of m_i(s): both tiles' rows are
      // reduced in the CTA, then one atomic per (h, s, k)
      for (int s0 = 0; s0 <= it.k; s0 += 16) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = (row_ok && s0 + i <= it.k) ? mrow[(s0 + i) * kBlockM] * inv_l : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
        }
        if (lane < 16 && s0 + lane <= it.k) {
          float mine = v[0];
#pragma unroll
          for (int i = 1; i < 16; ++i) mine = (lane == i) ? v[i] : mine;
          red_sm[(x * 4 + (warp & 3)) * 32 + s0 + lane] = mine;
        }
      }
      named_bar_sync(1, 2 * kBlockM);
      if (x == 0 && r <= it.k && *abort_flag == 0) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) tot += red_sm[w * 32 + r];
        const float inv_rows = 1.f / (float(p.B) * float(p.sc.n[it.k]));
        atomicAdd(p.mass + (int64_t(it.h) * p.sc.S + r) * p.sc.S + it.k, tot * inv_rows);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
static int encode_dense(CUtensorMap* m, const uint16_t* base, int D, int64_t rows, int64_t planes) {
  const uint64_t dims[3] = {uint64_t(D), uint64_t(rows), uint64_t(planes)};
  const uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(rows) * D * 2};
  return encode_bf16_map(m, base, 3, dims, strides, 128);
}
static int encode_rows(CUtensorMap* m, const uint16_t* base, int D, int64_t rows) {
  const uint64_t dims[2] = {uint64_t(D), uint64_t(rows)};
  const uint64_t strides[1] = {uint64_t(D) * 2};
  return encode_bf16_map(m, base, 2, dims, strides, 128);
}

// Query-tile pairs (256 rows of one scale) of the selected scales, heaviest
// (most keys) first within each (batch, head).
static int build_qtiles(Params& p, int query_scale) {
  struct E { int64_t w; uint32_t v; };
  std::vector<E> e;
  for (int k = 0; k < p.sc.S; ++k) {
    if (query_scale >= 0 && k != query_scale) continue;
    for (int r = 0; r < p.sc.n[k]; r += 2 * kBlockM)
      e.push_back({int64_t(p.sc.off[k]) + p.sc.n[k], (uint32_t(k) << 24) | uint32_t(r)});
  }
  if (e.empty() || int(e.size()) > kMaxPairs) return VARK_E_SHAPE;
  std::stable_sort(e.begin(), e.end(), [](const E& a, const E& b) { return a.w > b.w; });
  p.n_pairs = int(e.size());
  for (int i = 0; i < p.n_pairs; ++i) p.pair[i] = e[i].v;
  return VARK_OK;
}

// Failure-detection test hook: VARK_TEST_WAIT_LIMIT_MS shortens the bounded
// waits, VARK_TEST_WITHHOLD_KV_TILE=j makes every CTA's producer stop before
// key tile j so the waits on it run out (the kernel then reports
// VARK_E_TIMEOUT through the status word).  Both unset in normal use.
static void apply_test_hooks(Params& p) {
  p.wait_limit_ns = kWaitLimitNs;
  p.withhold_tile = -1;
  if (const char* e = std::getenv("VARK_TEST_WAIT_LIMIT_MS")) {
    const long ms = std::strtol(e, nullptr, 10);
    if (ms > 0 && ms <= 10000) p.wait_limit_ns = uint64_t(ms) * 1000000ull;
  }
  if (const char* e = std::getenv("VARK_TEST_WITHHOLD_KV_TILE")) {
    const long j = std::strtol(e, nullptr, 10);
    if (j >= 0 && j < (1 << 20)) p.withhold_tile = int(j);
  }
}

template <int D, bool PRUNED, bool MASS, bool WITH_O = true, int QB = 0>
static int launch(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& kc,
                  const CUtensorMap& vc, Params& p, cudaStream_t st) {
  apply_test_hooks(p);
  auto kern = attn_kernel<D, PRUNED, MASS, WITH_O, QB>;
  const int smem = Smem<D, QB>::alloc(MASS, p.sc.S);
  if (smem > kMaxSmemOptin) return VARK_E_SHAPE;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return VARK_E_CUDA;
  }
  const int64_t grid = int64_t(p.n_pairs) * p.B * p.H;
  if (grid > INT32_MAX) return VARK_E_SHAPE;
  kern<<<unsigned(grid), kThreads, smem, st>>>(q, k, v, kc, vc, p);
  return cudaGetLastError() == cudaSuccess ? VARK_OK : VARK_E_CUDA;
}

static bool finite_shape(int B, int H, int T, int D) {
  return B >= 1 && H >= 1 && int64_t(B) * H <= INT32_MAX / 2 && int64_t(B) * H * T * D < (int64_t(1) << 40);
}

}  // namespace attn
}  // namespace vark

using namespace vark;
using namespace vark::attn;

extern "C" int vark_scas_accumulate(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int H, int D,
                                    int S, const int32_t* sides, const float* tau, const float* bias, float* mass,
                                    uint16_t* out, int32_t* dev_status, void* stream) {
  if (!q || !k || !v || !tau || !mass || !dev_status) return VARK_E_ARG;
  Params lp;
  int rc = make_scale_table(S, sides, &lp.sc);
  if (rc) return rc;
  if (D != 64 && D != 128) return VARK_E_SHAPE;
  if (!finite_shape(B, H, lp.sc.T, D)) return VARK_E_SHAPE;
  // the per-row mass partials of every scale must fit next to the tiles
  if ((D == 128 ? Smem<128>::alloc(true, S) : Smem<64>::alloc(true, S)) > kMaxSmemOptin) return VARK_E_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (out && !aligned16(out))) return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  lp.B = B; lp.H = H;
  lp.scale_log2 = kLog2e / sqrtf(float(D));
  lp.tau = tau; lp.bias = bias; lp.mass = mass; lp.out = out; lp.status = dev_status;
  lp.q_rows = lp.sc.T; lp.q_scale_rows = 0; lp.local_scale_only = 0;
  lp.R_l = 0; lp.head_off = nullptr; lp.seg_off = nullptr; lp.past_len = nullptr;
  lp.kq = lp.vq = lp.ktab = lp.vtab = nullptr; lp.kc_rows = 0;
  if ((rc = build_qtiles(lp, -1))) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = encode_dense(&tq, q, D, lp.sc.T, int64_t(B) * H))) return rc;
  if ((rc = encode_dense(&tk, k, D, lp.sc.T, int64_t(B) * H))) return rc;
  if ((rc = encode_dense(&tv, v, D, lp.sc.T, int64_t(B) * H))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (out == nullptr)   // S-CAS only: no V, no PV
    return D == 128 ? launch<128, false, true, false>(tq, tk, tv, tk, tv, lp, st)
                    : launch<64, false, true, false>(tq, tk, tv, tk, tv, lp, st);
  return D == 128 ? launch<128, false, true>(tq, tk, tv, tk, tv, lp, st)
                  : launch<64, false, true>(tq, tk, tv, tk, tv, lp, st);
}

// The packed past of a quantised cache (null: bf16 past in kc / vc).
struct PackedPast {
  int bits;                 // 8, 4 or 3
  const void* kq;
  const void* vq;
  const void* ktab;
  const void* vtab;
};

static int pruned_common(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, int64_t kc_rows,
                         const uint16_t* k_local, const uint16_t* v_local, int B, int H, int S, int D,
                         const int32_t* sides, int query_scale, bool local_scale_only, const int32_t* head_off,
                         const int32_t* seg_off, const int32_t* past_len, const float* tau, const float* bias,
                         uint16_t* out, int32_t* dev_status, void* stream, const PackedPast* packed = nullptr) {
  if (!q || !k_local || !v_local || !head_off || !seg_off || !past_len || !tau || !out || !dev_status)
    return VARK_E_ARG;
  if (kc_rows < 0) return VARK_E_ARG;
  if (packed) {
    if (kc_rows > 0 && (!packed->kq || !packed->vq || !packed->ktab || !packed->vtab)) return VARK_E_ARG;
  } else if (kc_rows > 0 && (!kc || !vc)) {
    return VARK_E_ARG;
  }
  Params lp;
  int rc = make_scale_table(S, sides, &lp.sc);
  if (rc) return rc;
  if (D != 64 && D != 128) return VARK_E_SHAPE;
  // a packed K/V tile is copied whole: its rows must be a multiple of 16 bytes
  if (packed && (D * packed->bits / 8) % 16 != 0) return VARK_E_SHAPE;
  if (query_scale < -1 || query_scale >= S || (local_scale_only && query_scale < 0)) return VARK_E_ARG;
  if (!finite_shape(B, H, lp.sc.T, D)) return VARK_E_SHAPE;
  if (kc_rows % B != 0 || kc_rows > INT32_MAX) return VARK_E_SHAPE;
  if (!aligned16(q) || !aligned16(k_local) || !aligned16(v_local) || !aligned16(out)) return VARK_E_ALIGN;
  if (kc_rows > 0 && !packed && (!aligned16(kc) || !aligned16(vc))) return VARK_E_ALIGN;
  if (kc_rows > 0 && packed &&
      (!aligned16(packed->kq) || !aligned16(packed->vq) || !aligned16(packed->ktab) || !aligned16(packed->vtab)))
    return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  lp.B = B; lp.H = H;
  lp.scale_log2 = kLog2e / sqrtf(float(D));
  lp.tau = tau; lp.bias = bias; lp.mass = nullptr; lp.out = out; lp.status = dev_status;
  lp.q_rows = query_scale < 0 ? lp.sc.T : lp.sc.n[query_scale];
  lp.q_scale_rows = query_scale < 0 ? 0 : 1;
  lp.local_scale_only = local_scale_only ? 1 : 0;
  lp.R_l = kc_rows / B;
  lp.head_off = head_off; lp.seg_off = seg_off; lp.past_len = past_len;
  lp.kq = packed ? packed->kq : nullptr;
  lp.vq = packed ? packed->vq : nullptr;
  lp.ktab = packed ? packed->ktab : nullptr;
  lp.vtab = packed ? packed->vtab : nullptr;
  lp.kc_rows = kc_rows;
  if ((rc = build_qtiles(lp, query_scale))) return rc;
  const int64_t local_rows = local_scale_only ? lp.sc.n[query_scale] : lp.sc.T;
  CUtensorMap tq, tk, tv, tkc, tvc;
  if ((rc = encode_dense(&tq, q, D, lp.q_rows, int64_t(B) * H))) return rc;
  if ((rc = encode_dense(&tk, k_local, D, local_rows, int64_t(B) * H))) return rc;
  if ((rc = encode_dense(&tv, v_local, D, local_rows, int64_t(B) * H))) return rc;
  if (kc_rows > 0 && !packed) {
    if ((rc = encode_rows(&tkc, kc, D, kc_rows))) return rc;
    if ((rc = encode_rows(&tvc, vc, D, kc_rows))) return rc;
  } else {
    // No head keeps past rows, or the past comes as packed codes: these maps
    // are never read; they only need to be valid 2-D maps.
    if ((rc = encode_rows(&tkc, k_local, D, 1))) return rc;
    if ((rc = encode_rows(&tvc, v_local, D, 1))) return rc;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (packed && kc_rows > 0) {
    switch (packed->bits * 1000 + D) {
      case 8128: return launch<128, true, false, true, 8>(tq, tk, tv, tkc, tvc, lp, st);
      case 8064: return launch<64, true, false, true, 8>(tq, tk, tv, tkc, tvc, lp, st);
      case 4128: return launch<128, true, false, true, 4>(tq, tk, tv, tkc, tvc, lp, st);
      case 4064: return launch<64, true, false, true, 4>(tq, tk, tv, tkc, tvc, lp, st);
      case 3128: return launch<128, true, false, true, 3>(tq, tk, tv, tkc, tvc, lp, st);
      default: return VARK_E_SHAPE;
    }
  }
  return D == 128 ? launch<128, true, false>(tq, tk, tv, tkc, tvc, lp, st)
                  : launch<64, true, false>(tq, tk, tv, tkc, tvc, lp, st);
}

extern "C" int vark_pruned_attention(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, int64_t kc_rows,
                                     const uint16_t* k_dense, const uint16_t* v_dense, int B, int H, int S, int D,
                                     const int32_t* sides, int query_scale, const int32_t* head_off,
                                     const int32_t* seg_off, const int32_t* past_len, const float* tau,
                                     const float* bias, uint16_t* out, int32_t* dev_status, void* stream) {
  return pruned_common(q, kc, vc, kc_rows, k_dense, v_dense, B, H, S, D, sides, query_scale, false, head_off,
                       seg_off, past_len, tau, bias, out, dev_status, stream);
}

extern "C" int vark_pruned_attention_step(const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                          int64_t kc_rows, const uint16_t* k_local, const uint16_t* v_local, int B,
                                          int H, int S, int D, const int32_t* sides, int scale,
                                          const int32_t* head_off, const int32_t* seg_off, const int32_t* past_len,
                                          const float* tau, const float* bias, uint16_t* out, int32_t* dev_status,
                                          void* stream) {
  if (scale < 0) return VARK_E_ARG;
  return pruned_common(q, kc, vc, kc_rows, k_local, v_local, B, H, S, D, sides, scale, true, head_off, seg_off,
                       past_len, tau, bias, out, dev_status, stream);
}

// Pruned attention over a quantised retained cache: the past K/V of this
// layer come as packed codes plus per-(batch, head, scale, channel) tables and
// are dequantised inside the kernel; no bf16 copy of the cache is written.
static int pruned_packed(int bits, const uint16_t* q, const void* kq, const void* vq, const void* ktab,
                         const void* vtab, int64_t kc_rows, const uint16_t* k_dense, const uint16_t* v_dense, int B,
                         int H, int S, int D, const int32_t* sides, int query_scale, const int32_t* head_off,
                         const int32_t* seg_off, const int32_t* past_len, const float* tau, const float* bias,
                         uint16_t* out, int32_t* dev_status, void* stream) {
  const PackedPast pk = {bits, kq, vq, ktab, vtab};
  return pruned_common(q, nullptr, nullptr, kc_rows, k_dense, v_dense, B, H, S, D, sides, query_scale, false,
                       head_off, seg_off, past_len, tau, bias, out, dev_status, stream, &pk);
}

extern "C" int vark_pruned_attention_int8(const uint16_t* q, const int8_t* kq, const int8_t* vq,
                                          const float* k_absmax, const float* v_absmax, int64_t kc_rows,
                                          const uint16_t* k_dense, const uint16_t* v_dense, int B, int H, int S,
                                          int D, const int32_t* sides, int query_scale, const int32_t* head_off,
                                          const int32_t* seg_off, const int32_t* past_len, const float* tau,
                                          const float* bias, uint16_t* out, int32_t* dev_status, void* stream) {
  return pruned_packed(8, q, kq, vq, k_absmax, v_absmax, kc_rows, k_dense, v_dense, B, H, S, D, sides, query_scale,
                       head_off, seg_off, past_len, tau, bias, out, dev_status, stream);
}

extern "C" int vark_pruned_attention_int4(const uint16_t* q, const uint8_t* kq, const uint8_t* vq,
                                          const uint16_t* k_scale, const uint16_t* v_scale, int64_t kc_rows,
                                          const uint16_t* k_dense, const uint16_t* v_dense, int B, int H, int S,
                                          int D, const int32_t* sides, int query_scale, const int32_t* head_off,
                                          const int32_t* seg_off, const int32_t* past_len, const float* tau,
                                          const float* bias, uint16_t* out, int32_t* dev_status, void* stream) {
  return pruned_packed(4, q, kq, vq, k_scale, v_scale, kc_rows, k_dense, v_dense, B, H, S, D, sides, query_scale,
                       head_off, seg_off, past_len, tau, bias, out, dev_status, stream);
}

extern "C" int vark_pruned_attention_int3(const uint16_t* q, const uint8_t* kq, const uint8_t* vq,
                                          const uint16_t* k_scale, const uint16_t* v_scale, int64_t kc_rows,
                                          const uint16_t* k_dense, const uint16_t* v_dense, int B, int H, int S,
                                          int D, const int32_t* sides, int query_scale, const int32_t* head_off,
                                          const int32_t* seg_off, const int32_t* past_len, const float* tau,
                                          const float* bias, uint16_t* out, int32_t* dev_status, void* stream) {
  return pruned_packed(3, q, kq, vq, k_scale, v_scale, kc_rows, k_dense, v_dense, B, H, S, D, sides, query_scale,
                       head_off, seg_off, past_len, tau, bias, out, dev_status, stream);
}
