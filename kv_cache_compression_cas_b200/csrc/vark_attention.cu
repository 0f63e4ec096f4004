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
// One CTA computes one 128-row query tile of one (batch, head) over a list of
// 128-key tiles.  Roles (256 threads):
//   warp 0      TMA producer: Q once, then K/V tiles into a 2-stage ring;
//   warp 1      owns TMEM (512 columns) and issues tcgen05.mma from one thread:
//               S_j = Q K_j^T into one of two TMEM S buffers (one tile ahead),
//               then O += P_j V_j into the TMEM O accumulator;
//   warps 4..7  softmax, one thread per query row (TMEM lane = row): read S_j
//               with tcgen05.ld, online softmax in the exp2 domain, write P_j
//               as bf16 into shared memory in the 128-byte-swizzled K-major
//               operand layout, rescale O in TMEM only when the running max
//               grows by more than 2^8 (the stale max cancels in O / l).
// Operands: Q, K, P K-major SW128; V MN-major SW128 (as stored, [key][d]).
// Every mbarrier wait is bounded: on timeout the kernel records
// VARK_E_TIMEOUT in the caller's status word, drains its own async work with
// bounded waits, frees TMEM and returns.
#include <algorithm>
#include <vector>

#include "vark_common.cuh"

namespace vark {
namespace attn {

constexpr int kThreads = 256;
constexpr int kBlockM = 128;
constexpr int kBlockN = 128;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxQTiles = 512;
constexpr int kPanelBytes = 128 * 128;   // 128 rows x 128 bytes (64 bf16)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 domain

struct Params {
  ScaleTable sc;
  int B, H;
  int n_qt;                       // query-tile kinds per (batch, head)
  uint32_t qt[kMaxQTiles];        // (scale << 24) | row start within the scale
  float scale_log2;               // log2(e) / sqrt(D)
  const float* tau;
  const float* bias;              // [H][S] or null
  float* mass;                    // [H][S][S] (calibration)
  uint16_t* out;                  // same layout as q, or null
  int32_t* status;
  int q_rows;                     // rows per (b, h) of q / out
  int q_scale_rows;               // 1: q row = row within scale (single-scale q)
  // pruned attention
  int64_t R_l;
  const int32_t* head_off;        // [H]
  const int32_t* seg_off;         // [H][S]
  const int32_t* past_len;        // [H][S]
};

template <int D>
struct Smem {
  static constexpr int kQPanels = D / 64;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kQPanels * kPanelBytes;
  static constexpr int kV = kK + kStages * kQPanels * kPanelBytes;
  static constexpr int kP = kV + kStages * kQPanels * kPanelBytes;
  static constexpr int kMass = kP + 2 * kPanelBytes;                     // [S][128] fp32
  static constexpr int kRed = kMass + VARK_MAX_SCALES * kBlockM * 4;     // [4][32] fp32
  static constexpr int kBar = kRed + 4 * 32 * 4;
  // barriers: q, k_full[2], v_full[2], kv_empty[2], s_full[2], s_free[2], p_full, o_done, drain
  static constexpr int kNumBars = 1 + 2 * kStages + kStages + 2 + 2 + 3;
  static constexpr int kMisc = kBar + kNumBars * 8;                       // tmem base, abort flag
  static constexpr int kTotal = kMisc + 16;
  static constexpr int kAlloc = kTotal + 1024;                            // alignment slack
};

// Tile of keys j of one work item.
struct KTile {
  int src;        // 0: dense K/V ([B*H][T][D] map), 1: compacted K/V ([rows][D] map)
  int row;        // first row (dense: within (b,h); compacted: absolute)
  int valid;      // valid key columns in this tile
  int key0;       // first key index in the item's key list
};

template <bool PRUNED>
struct Item {
  int b, h, bh, k, qrow0, rows_valid;
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
      t.row = p.sc.off[k] + jj * kBlockN;
      t.valid = min(kBlockN, p.sc.n[k] - jj * kBlockN);
      t.key0 = jj * kBlockN;
    }
    return t;
  }
};

template <bool PRUNED>
__device__ Item<PRUNED> decode_item(const Params& p) {
  Item<PRUNED> it;
  const int BH = p.B * p.H;
  const int kind = blockIdx.x / BH;
  it.bh = blockIdx.x % BH;
  it.b = it.bh / p.H;
  it.h = it.bh % p.H;
  const uint32_t e = p.qt[kind];
  it.k = int(e >> 24);
  it.qrow0 = int(e & 0xFFFFFFu);
  it.rows_valid = min(kBlockM, p.sc.n[it.k] - it.qrow0);
  if (!PRUNED) {
    const int Lk = p.sc.off[it.k] + p.sc.n[it.k];
    it.n_tiles = (Lk + kBlockN - 1) / kBlockN;
    it.n_past = 0;
    it.past = 0;
    it.kc_row0 = 0;
  } else {
    it.past = p.past_len[it.h * p.sc.S + it.k];
    it.n_past = (it.past + kBlockN - 1) / kBlockN;
    it.n_tiles = it.n_past + (p.sc.n[it.k] + kBlockN - 1) / kBlockN;
    it.kc_row0 = int64_t(it.b) * p.R_l + p.head_off[it.h];
  }
  return it;
}

// Calls f(col_begin, col_end, scale) for every source-scale segment of the
// valid columns of a key tile, in column order.
template <bool PRUNED, typename F>
__device__ __forceinline__ void for_each_segment(const Params& p, const Item<PRUNED>& it, const KTile& t, F&& f) {
  if (!PRUNED) {
    const int lo = t.key0, hi = t.key0 + t.valid;
    for (int s = 0; s <= it.k; ++s) {
      const int a = max(p.sc.off[s], lo), e = min(p.sc.off[s] + p.sc.n[s], hi);
      if (a < e) f(a - lo, e - lo, s);
    }
  } else if (t.src == 1) {
    const int lo = t.key0, hi = t.key0 + t.valid;
    for (int s = 0; s < it.k; ++s) {
      const int so = p.seg_off[it.h * p.sc.S + s];
      if (so < 0) continue;
      const int a = max(so, lo), e = min(so + p.sc.n[s], hi);
      if (a < e) f(a - lo, e - lo, s);
    }
  } else {
    f(0, t.valid, it.k);
  }
}

template <int D, bool PRUNED, bool MASS>
__global__ void __launch_bounds__(kThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
            const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
            const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ Params p) {
  using L = Smem<D>;
  constexpr int QP = L::kQPanels;
  constexpr uint32_t kTileBytes = QP * kPanelBytes;   // one Q / K / V tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + L::kQ, sK = sbase + L::kK, sV = sbase + L::kV, sP = sbase + L::kP;
  float* mass_sm = reinterpret_cast<float*>(smem + L::kMass);
  float* red_sm = reinterpret_cast<float*>(smem + L::kRed);
  const uint32_t bar0 = sbase + L::kBar;
  const uint32_t bar_q = bar0;
  auto bar_k_full = [&](int s) { return bar0 + 8 * (1 + s); };
  auto bar_v_full = [&](int s) { return bar0 + 8 * (1 + kStages + s); };
  auto bar_kv_empty = [&](int s) { return bar0 + 8 * (1 + 2 * kStages + s); };
  auto bar_s_full = [&](int b) { return bar0 + 8 * (1 + 3 * kStages + b); };
  auto bar_s_free = [&](int b) { return bar0 + 8 * (3 + 3 * kStages + b); };
  const uint32_t bar_p_full = bar0 + 8 * (5 + 3 * kStages);
  const uint32_t bar_o_done = bar0 + 8 * (6 + 3 * kStages);
  const uint32_t bar_drain = bar0 + 8 * (7 + 3 * kStages);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Item<PRUNED> it = decode_item<PRUNED>(p);
  const int n = it.n_tiles;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_k_full(s), 1);
      mbar_init(bar_v_full(s), 1);
      mbar_init(bar_kv_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_s_full(b), 1);
      mbar_init(bar_s_free(b), kBlockM);
    }
    mbar_init(bar_p_full, kBlockM);
    mbar_init(bar_o_done, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_S0 = tmem, tmem_O = tmem + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (PRUNED) {
        tma_prefetch_desc(&tm_kc);
        tma_prefetch_desc(&tm_vc);
      }
      const int qrow = (p.q_scale_rows ? 0 : p.sc.off[it.k]) + it.qrow0;
      mbar_arrive_expect_tx(bar_q, kTileBytes);
      for (int c = 0; c < QP; ++c) tma_load_3d(sQ + c * kPanelBytes, &tm_q, bar_q, c * 64, qrow, it.bh);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % kStages;
        if (j >= kStages && !mbar_wait(bar_kv_empty(st), ((j / kStages) - 1) & 1, abort_flag, p.status)) break;
        const KTile t = it.tile(p, j);
        mbar_arrive_expect_tx(bar_k_full(st), kTileBytes);
        for (int c = 0; c < QP; ++c) {
          const uint32_t dst = sK + (st * QP + c) * kPanelBytes;
          if (t.src == 0) tma_load_3d(dst, &tm_k, bar_k_full(st), c * 64, t.row, it.bh);
          else tma_load_2d(dst, &tm_kc, bar_k_full(st), c * 64, t.row);
        }
        mbar_arrive_expect_tx(bar_v_full(st), kTileBytes);
        for (int c = 0; c < QP; ++c) {
          const uint32_t dst = sV + (st * QP + c) * kPanelBytes;
          if (t.src == 0) tma_load_3d(dst, &tm_v, bar_v_full(st), c * 64, t.row, it.bh);
          else tma_load_2d(dst, &tm_vc, bar_v_full(st), c * 64, t.row);
        }
        issued = j + 1;
      }
      // Drain: every load this thread issued has landed before the CTA exits
      // (immediate on the normal path; bounded on the abort path).
      volatile int no_abort = 0;
      mbar_wait(bar_q, 0, &no_abort, p.status);
      for (int j = max(0, issued - kStages); j < issued; ++j) {
        mbar_wait(bar_k_full(j % kStages), (j / kStages) & 1, &no_abort, p.status);
        mbar_wait(bar_v_full(j % kStages), (j / kStages) & 1, &no_abort, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, false, true);
      bool ok = mbar_wait(bar_q, 0, abort_flag, p.status);
      auto issue_s = [&](int j) -> bool {
        const int st = j % kStages, sb = j & 1;
        if (!mbar_wait(bar_k_full(st), (j / kStages) & 1, abort_flag, p.status)) return false;
        if (j >= 2 && !mbar_wait(bar_s_free(sb), ((j >> 1) - 1) & 1, abort_flag, p.status)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
          const uint64_t a = smem_desc_sw128(sQ + off, 16, 1024);
          const uint64_t b = smem_desc_sw128(sK + st * kTileBytes + off, 16, 1024);
          mma_bf16_ss(tmem_S0 + sb * kBlockN, a, b, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar_s_full(sb));
        return true;
      };
      if (ok && n > 0) ok = issue_s(0);
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n && !(ok = issue_s(j + 1))) break;
        const int st = j % kStages;
        if (!(ok = mbar_wait(bar_p_full, j & 1, abort_flag, p.status))) break;
        if (!(ok = mbar_wait(bar_v_full(st), (j / kStages) & 1, abort_flag, p.status))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          const uint64_t a = smem_desc_sw128(sP + (kk >> 2) * kPanelBytes + (kk & 3) * 32, 16, 1024);
          const uint64_t b = smem_desc_sw128(sV + st * kTileBytes + kk * 2048, kPanelBytes, 1024);
          mma_bf16_ss(tmem_O, a, b, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar_o_done);
        if (j + kStages < n) mma_commit(bar_kv_empty(st));
      }
      // Drain: all MMAs of this thread complete before TMEM is released.
      mma_commit(bar_drain);
      volatile int no_abort = 0;
      mbar_wait(bar_drain, 0, &no_abort, p.status);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x - 128;                 // query row = TMEM lane
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const float qk2 = p.tau[it.h] * p.scale_log2;
    const float* bias_h = p.bias ? p.bias + it.h * p.sc.S : nullptr;
    float m_used = -INFINITY, l_sum = 0.f;
    if (MASS)
      for (int s = 0; s < p.sc.S; ++s) mass_sm[s * kBlockM + r] = 0.f;
    bool ok = true;
    const uint32_t prow = uint32_t(r) * 128u;
    const uint32_t rsw = uint32_t(r & 7);

    for (int j = 0; j < n; ++j) {
      const int sb = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar_s_full(sb), (j >> 1) & 1, abort_flag, p.status));
      if (!ok) break;
      tc_fence_after();
      float x[kBlockN];
      {
        uint32_t v[kBlockN / 32][32];
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) tmem_ld32(tmem_S0 + sb * kBlockN + c * 32 + lane_base, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kBlockN / 32; ++c) {
          reg_fence32(v[c]);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[c * 32 + i] = __uint_as_float(v[c][i]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_s_free(sb));

      const KTile t = it.tile(p, j);
      // logits in the log2 domain, bias per source-scale segment, mask tail
      int nseg = 0, seg_scale = 0;
      for_each_segment<PRUNED>(p, it, t, [&](int, int, int s) { ++nseg; seg_scale = s; });
      if (nseg == 1) {
        const float b2 = bias_h ? bias_h[seg_scale] * kLog2e : 0.f;
#pragma unroll
        for (int c = 0; c < kBlockN; ++c) x[c] = (c < t.valid) ? fmaf(x[c], qk2, b2) : -INFINITY;
      } else {
#pragma unroll
        for (int c = 0; c < kBlockN; ++c) x[c] = (c < t.valid) ? x[c] * qk2 : -INFINITY;
        if (bias_h) {
          for_each_segment<PRUNED>(p, it, t, [&](int cb, int ce, int s) {
            const float b2 = bias_h[s] * kLog2e;
#pragma unroll
            for (int c = 0; c < kBlockN; ++c) x[c] += (c >= cb && c < ce) ? b2 : 0.f;
          });
        }
      }
      float m_tile = x[0];
#pragma unroll
      for (int c = 1; c < kBlockN; ++c) m_tile = fmaxf(m_tile, x[c]);

      // PV_{j-1} complete: the P buffer is free and O is stable.
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done, (j - 1) & 1, abort_flag, p.status));
        if (!ok) break;
      }
      // Rescale when this row's max grew past the threshold; the TMEM access
      // is warp-collective, so a warp rescales if any of its rows must.
      bool rescaled = false;
      float f = 1.f;
      if (j == 0) {
        m_used = m_tile;
      } else if (m_tile > m_used + kRescaleThreshold) {
        f = ex2_approx(m_used - m_tile);
        m_used = m_tile;
        l_sum *= f;
        if (MASS)
          for (int s = 0; s <= it.k; ++s) mass_sm[s * kBlockM + r] *= f;
      }
      if (j > 0 && __any_sync(0xffffffffu, f != 1.f)) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem_O + c * 32 + lane_base, v);
          tmem_wait_ld();
          reg_fence32(v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
          tmem_st32(tmem_O + c * 32 + lane_base, v);
        }
        rescaled = true;
      }
      float tile_sum = 0.f;
#pragma unroll
      for (int c = 0; c < kBlockN; ++c) {
        x[c] = ex2_approx(x[c] - m_used);
        tile_sum += x[c];
      }
      l_sum += tile_sum;
      if (MASS) {
        if (nseg == 1) {
          mass_sm[seg_scale * kBlockM + r] += tile_sum;
        } else {
          for_each_segment<PRUNED>(p, it, t, [&](int cb, int ce, int s) {
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < kBlockN; ++c) acc += (c >= cb && c < ce) ? x[c] : 0.f;
            mass_sm[s * kBlockM + r] += acc;
          });
        }
      }
      // P row -> shared memory, 128-byte swizzled K-major operand layout
#pragma unroll
      for (int q = 0; q < kBlockN / 8; ++q) {
        const uint32_t addr = sP + (q >> 3) * kPanelBytes + prow + ((uint32_t(q & 7) ^ rsw) << 4);
        const uint32_t w0 = pack_bf16x2(x[8 * q + 0], x[8 * q + 1]);
        const uint32_t w1 = pack_bf16x2(x[8 * q + 2], x[8 * q + 3]);
        const uint32_t w2 = pack_bf16x2(x[8 * q + 4], x[8 * q + 5]);
        const uint32_t w3 = pack_bf16x2(x[8 * q + 6], x[8 * q + 7]);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                     : "memory");
      }
      fence_proxy_async_smem();
      if (rescaled) tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p_full);
    }

    // ---------------------------------------------------------- epilogue
    if (ok && n > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar_o_done, (n - 1) & 1, abort_flag, p.status));
    const bool row_ok = ok && r < it.rows_valid;
    const float inv_l = 1.f / l_sum;
    if (ok && p.out != nullptr) {
      tc_fence_after();
      const int out_row = (p.q_scale_rows ? 0 : p.sc.off[it.k]) + it.qrow0 + r;
      uint16_t* orow = p.out + (int64_t(it.bh) * p.q_rows + out_row) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem_O + c * 32 + lane_base, v);
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
      // mean over the B * n_k rows of scale k of m_i(s), one atomic per (h, s, k)
      const float inv_rows = 1.f / (float(p.B) * float(p.sc.n[it.k]));
      for (int s = 0; s <= it.k; ++s) {
        float v = row_ok ? mass_sm[s * kBlockM + r] * inv_l : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red_sm[(warp & 3) * 32 + s] = v;
      }
      named_bar_sync(1, kBlockM);
      if (ok && r <= it.k) {
        const float tot = red_sm[r] + red_sm[32 + r] + red_sm[64 + r] + red_sm[96 + r];
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

// Query-tile kinds of the selected scales, heaviest (most keys) first.
static int build_qtiles(Params& p, int query_scale) {
  struct E { int64_t w; uint32_t v; };
  std::vector<E> e;
  for (int k = 0; k < p.sc.S; ++k) {
    if (query_scale >= 0 && k != query_scale) continue;
    for (int r = 0; r < p.sc.n[k]; r += kBlockM) e.push_back({int64_t(p.sc.off[k]) + p.sc.n[k], (uint32_t(k) << 24) | uint32_t(r)});
  }
  if (e.empty() || int(e.size()) > kMaxQTiles) return VARK_E_SHAPE;
  std::stable_sort(e.begin(), e.end(), [](const E& a, const E& b) { return a.w > b.w; });
  p.n_qt = int(e.size());
  for (int i = 0; i < p.n_qt; ++i) p.qt[i] = e[i].v;
  return VARK_OK;
}

template <int D, bool PRUNED, bool MASS>
static int launch(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& kc,
                  const CUtensorMap& vc, const Params& p, cudaStream_t st) {
  auto kern = attn_kernel<D, PRUNED, MASS>;
  const int smem = Smem<D>::kAlloc;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    cudaGetLastError();
    return VARK_E_CUDA;
  }
  const int64_t grid = int64_t(p.n_qt) * p.B * p.H;
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
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || (out && !aligned16(out))) return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  lp.B = B; lp.H = H;
  lp.scale_log2 = kLog2e / sqrtf(float(D));
  lp.tau = tau; lp.bias = bias; lp.mass = mass; lp.out = out; lp.status = dev_status;
  lp.q_rows = lp.sc.T; lp.q_scale_rows = 0;
  lp.R_l = 0; lp.head_off = nullptr; lp.seg_off = nullptr; lp.past_len = nullptr;
  if ((rc = build_qtiles(lp, -1))) return rc;
  CUtensorMap tq, tk, tv;
  if ((rc = encode_dense(&tq, q, D, lp.sc.T, int64_t(B) * H))) return rc;
  if ((rc = encode_dense(&tk, k, D, lp.sc.T, int64_t(B) * H))) return rc;
  if ((rc = encode_dense(&tv, v, D, lp.sc.T, int64_t(B) * H))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch<128, false, true>(tq, tk, tv, tk, tv, lp, st)
                  : launch<64, false, true>(tq, tk, tv, tk, tv, lp, st);
}

extern "C" int vark_pruned_attention(const uint16_t* q, const uint16_t* kc, const uint16_t* vc, int64_t kc_rows,
                                     const uint16_t* k_dense, const uint16_t* v_dense, int B, int H, int S, int D,
                                     const int32_t* sides, int query_scale, const int32_t* head_off,
                                     const int32_t* seg_off, const int32_t* past_len, const float* tau,
                                     const float* bias, uint16_t* out, int32_t* dev_status, void* stream) {
  if (!q || !k_dense || !v_dense || !head_off || !seg_off || !past_len || !tau || !out || !dev_status)
    return VARK_E_ARG;
  if (kc_rows < 0 || (kc_rows > 0 && (!kc || !vc))) return VARK_E_ARG;
  Params lp;
  int rc = make_scale_table(S, sides, &lp.sc);
  if (rc) return rc;
  if (D != 64 && D != 128) return VARK_E_SHAPE;
  if (query_scale < -1 || query_scale >= S) return VARK_E_ARG;
  if (!finite_shape(B, H, lp.sc.T, D)) return VARK_E_SHAPE;
  if (kc_rows % B != 0 || kc_rows > INT32_MAX) return VARK_E_SHAPE;
  if (!aligned16(q) || !aligned16(k_dense) || !aligned16(v_dense) || !aligned16(out) ||
      (kc_rows > 0 && (!aligned16(kc) || !aligned16(vc))))
    return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  lp.B = B; lp.H = H;
  lp.scale_log2 = kLog2e / sqrtf(float(D));
  lp.tau = tau; lp.bias = bias; lp.mass = nullptr; lp.out = out; lp.status = dev_status;
  lp.q_rows = query_scale < 0 ? lp.sc.T : lp.sc.n[query_scale];
  lp.q_scale_rows = query_scale < 0 ? 0 : 1;
  lp.R_l = kc_rows / B;
  lp.head_off = head_off; lp.seg_off = seg_off; lp.past_len = past_len;
  if ((rc = build_qtiles(lp, query_scale))) return rc;
  CUtensorMap tq, tk, tv, tkc, tvc;
  if ((rc = encode_dense(&tq, q, D, lp.q_rows, int64_t(B) * H))) return rc;
  if ((rc = encode_dense(&tk, k_dense, D, lp.sc.T, int64_t(B) * H))) return rc;
  if ((rc = encode_dense(&tv, v_dense, D, lp.sc.T, int64_t(B) * H))) return rc;
  if (kc_rows > 0) {
    if ((rc = encode_rows(&tkc, kc, D, kc_rows))) return rc;
    if ((rc = encode_rows(&tvc, vc, D, kc_rows))) return rc;
  } else {
    // No head keeps past rows, so these maps are never read; they only need
    // to be valid 2-D maps.
    if ((rc = encode_rows(&tkc, k_dense, D, 1))) return rc;
    if ((rc = encode_rows(&tvc, v_dense, D, 1))) return rc;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch<128, true, false>(tq, tk, tv, tkc, tvc, lp, st)
                  : launch<64, true, false>(tq, tk, tv, tkc, tvc, lp, st);
}
