// Offset tables and cache compaction: apply a static keep[layer][head][scale]
// schedule by gathering the retained scale blocks of every (layer, batch,
// head) into the per-head ragged layout documented in vark.h.
// [HeatKV] project page, Method step 5: the static schedule is applied while
// scales are generated; the Abstract: allocation is head-specific.
//
// Compaction is a pure HBM stream (every retained byte read once and written
// once, dropped bytes never touched).  Work unit = (layer, batch, head, kept
// chunk of <= kChunkRows rows of one scale), walked in that (memory) order by
// one persistent grid.
// Each CTA first builds, in shared memory, the prefix of kept chunks over
// (layer, head) for its layer group, so a unit is found by one binary search
// and a walk over at most S scales.  Copies are 16-byte vectors, coalesced,
// with several loads in flight per thread before the stores.
#include <algorithm>
#include <type_traits>

#include "vark_common.cuh"

namespace vark {

// ---------------------------------------------------------------- offsets
struct OffsetsParams {
  ScaleTable sc;
  int L, H, B, D;
};

// One CTA.  head_off holds R[l][h] until the per-layer scan rewrites it, and
// layer_base[l+1] holds R_l until the layer scan; global writes are visible to
// the block after __syncthreads.
__global__ void __launch_bounds__(1024) offsets_kernel(const uint8_t* __restrict__ keep, OffsetsParams p,
                                                       int32_t* head_off, int32_t* seg_off, int32_t* past_len,
                                                       int64_t* layer_base) {
  const int LH = p.L * p.H;
  const int S = p.sc.S;
  for (int i = threadIdx.x; i < LH; i += blockDim.x) {
    int32_t running = 0;
    for (int s = 0; s < S; ++s) {
      past_len[i * S + s] = running;
      if (keep[i * S + s]) {
        seg_off[i * S + s] = running;
        running += p.sc.n[s];
      } else {
        seg_off[i * S + s] = -1;
      }
    }
    head_off[i] = running;
  }
  __syncthreads();
  for (int l = threadIdx.x; l < p.L; l += blockDim.x) {
    int64_t acc = 0;
    for (int h = 0; h < p.H; ++h) {
      const int32_t r = head_off[l * p.H + h];
      head_off[l * p.H + h] = int32_t(acc);
      acc += r;
    }
    layer_base[l + 1] = acc;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t base = 0;
    layer_base[0] = 0;
    for (int l = 0; l < p.L; ++l) {
      const int64_t rows = layer_base[l + 1];
      base += rows * p.B * p.D;
      layer_base[l + 1] = base;
    }
  }
}

// ---------------------------------------------------------------- compaction
// Exclusive scan of a[0, n) in shared memory by the whole block (kThreads
// threads, each owning a contiguous segment); a[n] receives the total.
template <int kThreads, int kMaxN>
__device__ __forceinline__ void block_exclusive_scan(int32_t* a, int n, int32_t* warp_tot) {
  constexpr int kPer = (kMaxN + kThreads - 1) / kThreads;
  const int seg0 = threadIdx.x * kPer;
  int32_t my_total = 0;
  for (int u = 0; u < kPer; ++u)
    if (seg0 + u < n) my_total += a[seg0 + u];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = my_total;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int32_t warp_base = 0, grand = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    if (w < warp) warp_base += warp_tot[w];
    grand += warp_tot[w];
  }
  int32_t run = warp_base + incl - my_total;
  for (int u = 0; u < kPer; ++u)
    if (seg0 + u < n) {
      const int32_t c = a[seg0 + u];
      a[seg0 + u] = run;
      run += c;
    }
  if (threadIdx.x == 0) a[n] = grand;
  __syncthreads();
}

constexpr int kChunkRows = 64;
constexpr int kCompactThreads = 256;
constexpr int kCompactInflight = 2;   // K + V vectors per thread in flight (2 measured ahead of 4 and 8)
constexpr int kMaxGroupLH = 4096;   // (layer, head) pairs per launch group

struct CompactParams {
  ScaleTable sc;
  int32_t chunks[VARK_MAX_SCALES];  // ceil(n_s / kChunkRows) for scales in [s_lo, s_hi), else 0
  int32_t src_off[VARK_MAX_SCALES]; // first source row of scale s inside a (b, h) block of the source
  int64_t src_rows;                 // rows per (b, h) block of the source (T, or n_k for one scale)
  int l0, nl;                       // layer group [l0, l0 + nl)
  int L, B, H, D;
  int64_t layer_stride;             // elements between source layers
  // compacted source (re-compaction): the source's own offset tables
  const int32_t* src_head_off;      // null: dense source
  const int32_t* src_seg_off;
  const int64_t* src_layer_base;
};

__global__ void __launch_bounds__(kCompactThreads, 4) compact_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, CompactParams p, const uint8_t* __restrict__ keep,
    const int32_t* __restrict__ head_off, const int32_t* __restrict__ seg_off, const int64_t* __restrict__ layer_base,
    uint4* __restrict__ kc, uint4* __restrict__ vc) {
  __shared__ int32_t chunk_prefix[kMaxGroupLH + 1];
  __shared__ uint32_t keep_mask[kMaxGroupLH];
  __shared__ int32_t warp_tot[kCompactThreads / 32];

  const int S = p.sc.S;
  const int H = p.H;
  const int nlh = p.nl * H;
  const int lh0 = p.l0 * H;

  // 1. kept-chunk count and keep bit mask of each (layer, head) of the group
  for (int i = threadIdx.x; i < nlh; i += kCompactThreads) {
    const uint8_t* kp = keep + int64_t(lh0 + i) * S;
    uint32_t m = 0;
    int32_t c = 0;
    for (int s = 0; s < S; ++s) {
      if (kp[s] && p.chunks[s] > 0) {
        m |= 1u << s;
        c += p.chunks[s];
      }
    }
    keep_mask[i] = m;
    chunk_prefix[i] = c;
  }
  __syncthreads();
  // 2. in-place exclusive scan; chunk_prefix[nlh] = total kept chunks
  block_exclusive_scan<kCompactThreads, kMaxGroupLH>(chunk_prefix, nlh, warp_tot);
  const int32_t grand = chunk_prefix[nlh];

  const int64_t units = int64_t(grand) * p.B;
  const int vec_per_row = p.D / 8;  // 16-byte vectors per row

  for (int64_t g = blockIdx.x; g < units; g += gridDim.x) {
    // Units in memory order (layer, batch, head, kept chunk): the CTAs in flight
    // read and write neighbouring addresses.  Layer: the last li with
    // B * chunk_prefix[li * H] <= g (empty layers are skipped by taking the last).
    int la = 0, lz = p.nl;
    while (lz - la > 1) {
      const int mid = (la + lz) >> 1;
      if (int64_t(chunk_prefix[mid * H]) * p.B <= g) la = mid; else lz = mid;
    }
    const int32_t c0 = chunk_prefix[la * H];
    const int32_t C = chunk_prefix[(la + 1) * H] - c0;
    const int64_t r = g - int64_t(c0) * p.B;
    const int b = int(r / C);
    const int32_t c = c0 + int32_t(r % C);
    // (layer, head) with chunk_prefix[i] <= c < chunk_prefix[i+1], inside layer la
    int lo = la * H, hi = (la + 1) * H;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (chunk_prefix[mid] <= c) lo = mid; else hi = mid;
    }
    const int i = lo;
    int32_t j = c - chunk_prefix[i];
    const uint32_t m = keep_mask[i];
    int s = 0;
    for (; s < S; ++s) {
      if (m >> s & 1u) {
        if (j < p.chunks[s]) break;
        j -= p.chunks[s];
      }
    }
    const int l = p.l0 + i / H;
    const int h = i % H;
    const int32_t r0 = j * kChunkRows;
    const int32_t nrows = min(kChunkRows, p.sc.n[s] - r0);
    const int64_t R_l = (layer_base[l + 1] - layer_base[l]) / (int64_t(p.B) * p.D);
    const int64_t dst_row = int64_t(b) * R_l + head_off[l * H + h] + seg_off[(l * H + h) * S + s] + r0;
    const int64_t dst_v = (layer_base[l] / 8) + dst_row * vec_per_row;
    int64_t src_v;
    if (p.src_head_off == nullptr) {
      const int64_t src_row = (int64_t(b) * H + h) * p.src_rows + p.src_off[s] + r0;
      src_v = (int64_t(l) * p.layer_stride) / 8 + src_row * vec_per_row;
    } else {
      const int32_t so = p.src_seg_off[(l * H + h) * S + s];
      if (so < 0) continue;   // not in the source: nothing to move
      const int64_t R_src = (p.src_layer_base[l + 1] - p.src_layer_base[l]) / (int64_t(p.B) * p.D);
      const int64_t src_row = int64_t(b) * R_src + p.src_head_off[l * H + h] + so + r0;
      src_v = p.src_layer_base[l] / 8 + src_row * vec_per_row;
    }
    const int nvec = nrows * vec_per_row;

    // kCompactInflight K + kCompactInflight V vectors in flight per thread, then the stores.
    for (int base = 0; base < nvec; base += kCompactInflight * kCompactThreads) {
      uint4 a[kCompactInflight], bq[kCompactInflight];
#pragma unroll
      for (int u = 0; u < kCompactInflight; ++u) {
        const int e = base + u * kCompactThreads + threadIdx.x;
        if (e < nvec) {
          a[u] = __ldcs(k + src_v + e);
          bq[u] = __ldcs(v + src_v + e);
        }
      }
#pragma unroll
      for (int u = 0; u < kCompactInflight; ++u) {
        const int e = base + u * kCompactThreads + threadIdx.x;
        if (e < nvec) {
          __stcs(kc + dst_v + e, a[u]);
          __stcs(vc + dst_v + e, bq[u]);
        }
      }
    }
  }
}

}  // namespace vark

using namespace vark;

extern "C" int vark_build_offsets(const uint8_t* keep, int L, int H, int S, const int32_t* sides, int B, int D,
                                  int32_t* head_off, int32_t* seg_off, int32_t* past_len, int64_t* layer_base,
                                  void* stream) {
  if (!keep || !head_off || !seg_off || !past_len || !layer_base) return VARK_E_ARG;
  OffsetsParams p;
  int rc = make_scale_table(S, sides, &p.sc);
  if (rc) return rc;
  if (L < 1 || H < 1 || B < 1 || D < 1) return VARK_E_SHAPE;
  if (int64_t(L) * H > 16384) return VARK_E_SHAPE;
  if (int64_t(B) * H * p.sc.T > INT32_MAX) return VARK_E_SHAPE;
  if (!aligned16(head_off) || !aligned16(seg_off) || !aligned16(past_len) || !aligned16(layer_base))
    return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  p.L = L; p.H = H; p.B = B; p.D = D;
  offsets_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(keep, p, head_off, seg_off, past_len, layer_base);
  return cudaGetLastError() == cudaSuccess ? VARK_OK : VARK_E_CUDA;
}

// Launches the gather for scales [s_lo, s_hi) of a source laid out per layer
// as [B][H][src_rows][D] with scale s starting at row src_off[s].
static int launch_gather(const uint16_t* k, const uint16_t* v, int64_t layer_stride, int L, int B, int H, int D,
                         CompactParams& p, int s_lo, int s_hi, int64_t src_rows, const int32_t* src_off,
                         const int32_t* src_head_off, const int32_t* src_seg_off, const int64_t* src_layer_base,
                         const uint8_t* keep, const int32_t* head_off, const int32_t* seg_off,
                         const int64_t* layer_base, uint16_t* kc, uint16_t* vc, cudaStream_t st) {
  p.L = L; p.B = B; p.H = H; p.D = D; p.layer_stride = layer_stride; p.src_rows = src_rows;
  p.src_head_off = src_head_off; p.src_seg_off = src_seg_off; p.src_layer_base = src_layer_base;
  for (int s = 0; s < VARK_MAX_SCALES; ++s) {
    const bool in = s < p.sc.S && s >= s_lo && s < s_hi;
    p.chunks[s] = in ? (p.sc.n[s] + kChunkRows - 1) / kChunkRows : 0;
    p.src_off[s] = in ? src_off[s] : 0;
  }
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int layers_per_group = std::max(1, kMaxGroupLH / H);
  for (int l0 = 0; l0 < L; l0 += layers_per_group) {
    p.l0 = l0;
    p.nl = std::min(layers_per_group, L - l0);
    compact_kernel<<<nsm * 4, kCompactThreads, 0, st>>>(reinterpret_cast<const uint4*>(k),
                                                        reinterpret_cast<const uint4*>(v), p, keep, head_off,
                                                        seg_off, layer_base, reinterpret_cast<uint4*>(kc),
                                                        reinterpret_cast<uint4*>(vc));
    if (cudaGetLastError() != cudaSuccess) return VARK_E_CUDA;
  }
  return VARK_OK;
}

extern "C" int vark_compact_kv(const uint16_t* k, const uint16_t* v, int64_t layer_stride, int L, int B, int H,
                               int S, int D, const int32_t* sides, const uint8_t* keep, const int32_t* head_off,
                               const int32_t* seg_off, const int64_t* layer_base, uint16_t* kc, uint16_t* vc,
                               void* stream) {
  if (!k || !v || !keep || !head_off || !seg_off || !layer_base || !kc || !vc) return VARK_E_ARG;
  CompactParams p;
  int rc = make_scale_table(S, sides, &p.sc);
  if (rc) return rc;
  if (L < 1 || H < 1 || B < 1 || D < 8 || D % 8 != 0 || D > 1024) return VARK_E_SHAPE;
  if (H > kMaxGroupLH) return VARK_E_SHAPE;
  if (layer_stride < int64_t(B) * H * p.sc.T * D) return VARK_E_ARG;
  if (layer_stride % 8 != 0) return VARK_E_ALIGN;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kc) || !aligned16(vc)) return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  return launch_gather(k, v, layer_stride, L, B, H, D, p, 0, S, p.sc.T, p.sc.off, nullptr, nullptr, nullptr, keep,
                       head_off, seg_off, layer_base, kc, vc, static_cast<cudaStream_t>(stream));
}

extern "C" int vark_append_scale(const uint16_t* k_new, const uint16_t* v_new, int64_t layer_stride, int L, int B,
                                 int H, int S, int D, const int32_t* sides, int scale, const uint8_t* keep,
                                 const int32_t* head_off, const int32_t* seg_off, const int64_t* layer_base,
                                 uint16_t* kc, uint16_t* vc, void* stream) {
  if (!k_new || !v_new || !keep || !head_off || !seg_off || !layer_base || !kc || !vc) return VARK_E_ARG;
  CompactParams p;
  int rc = make_scale_table(S, sides, &p.sc);
  if (rc) return rc;
  if (scale < 0 || scale >= S) return VARK_E_ARG;
  if (L < 1 || H < 1 || B < 1 || D < 8 || D % 8 != 0 || D > 1024) return VARK_E_SHAPE;
  if (H > kMaxGroupLH) return VARK_E_SHAPE;
  if (layer_stride < int64_t(B) * H * p.sc.n[scale] * D) return VARK_E_ARG;
  if (layer_stride % 8 != 0) return VARK_E_ALIGN;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kc) || !aligned16(vc)) return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  int32_t zero_off[VARK_MAX_SCALES] = {0};
  return launch_gather(k_new, v_new, layer_stride, L, B, H, D, p, scale, scale + 1, p.sc.n[scale], zero_off, nullptr,
                       nullptr, nullptr, keep, head_off, seg_off, layer_base, kc, vc,
                       static_cast<cudaStream_t>(stream));
}

extern "C" int vark_recompact_kv(const uint16_t* kc_old, const uint16_t* vc_old, const int32_t* head_off_old,
                                 const int32_t* seg_off_old, const int64_t* layer_base_old, int L, int B, int H,
                                 int S, int D, const int32_t* sides, int max_scale, const uint8_t* keep_new,
                                 const int32_t* head_off_new, const int32_t* seg_off_new,
                                 const int64_t* layer_base_new, uint16_t* kc_new, uint16_t* vc_new, void* stream) {
  if (!kc_old || !vc_old || !head_off_old || !seg_off_old || !layer_base_old || !keep_new || !head_off_new ||
      !seg_off_new || !layer_base_new || !kc_new || !vc_new)
    return VARK_E_ARG;
  if (kc_old == kc_new || vc_old == vc_new) return VARK_E_ARG;
  CompactParams p;
  int rc = make_scale_table(S, sides, &p.sc);
  if (rc) return rc;
  if (max_scale < 0 || max_scale > S) return VARK_E_ARG;
  if (L < 1 || H < 1 || B < 1 || D < 8 || D % 8 != 0 || D > 1024) return VARK_E_SHAPE;
  if (H > kMaxGroupLH) return VARK_E_SHAPE;
  if (!aligned16(kc_old) || !aligned16(vc_old) || !aligned16(kc_new) || !aligned16(vc_new)) return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  if (max_scale == 0) return VARK_OK;
  int32_t zero_off[VARK_MAX_SCALES] = {0};
  return launch_gather(kc_old, vc_old, 0, L, B, H, D, p, 0, max_scale, 0, zero_off, head_off_old, seg_off_old,
                       layer_base_old, keep_new, head_off_new, seg_off_new, layer_base_new, kc_new, vc_new,
                       static_cast<cudaStream_t>(stream));
}


// ---------------------------------------------------------------- int8 quantised retained cache
// [VAR-Q] summary page: groups indexed by (block, channel), block boundaries
// given by the generation loop, composable with eviction.  Here a block is one
// retained scale of one (layer, batch, head); every channel d of it has one
// absmax a; codes are rint(x / (a / 127)) clamped to [-127, 127] (IEEE fp32
// division, round half to even); x' = code * (a / 127).
//
// Quantisation reads every kept byte from HBM once.  A unit is one block of
// one tensor (K or V).  A block of at most kSmallRows rows (256 KB at D = 128)
// belongs to one CTA: a strided pass takes the channel maxima, a second pass
// over the same rows (still in L2) writes the codes.  A larger block is split over the
// kQuantCluster CTAs of a thread-block cluster: each CTA reduces its slice,
// the CTAs exchange partial maxima through distributed shared memory, then
// each writes the codes of its slice.  Channel maxima are taken on the bf16
// magnitude bits (non-negative bf16 values order like their bit patterns), two
// channels per 32-bit word.  Every absmax entry is written exactly once.

namespace vark {

constexpr int kQuantThreads = 128;
constexpr int kQuantCluster = 8;
constexpr int kQuantGroupLH = 2048;  // (layer, head) pairs per launch group
constexpr int kSmallRows = 1024;
constexpr int kQuantMaxD = 512;

struct QuantParams {
  ScaleTable sc;
  uint32_t big_mask;        // scales with n_s > kSmallRows
  int l0, nl;               // layer group [l0, l0 + nl)
  int L, B, H, D;
  int64_t layer_stride;     // elements between source layers
};

struct QBlock {
  int l, h, s, b, t;        // t: 0 = K, 1 = V
};

// Unit g of one size class: blocks of the class are numbered in memory order
// (layer, batch, head, kept scale), K and V of a block adjacent.
__device__ __forceinline__ QBlock decode_block(int64_t g, const int32_t* prefix, const uint32_t* masks,
                                               uint32_t cls, const QuantParams& p) {
  const int H = p.H;
  const int64_t two_b = 2 * int64_t(p.B);
  int la = 0, lz = p.nl;                      // last layer whose first unit is <= g
  while (lz - la > 1) {
    const int mid = (la + lz) >> 1;
    if (int64_t(prefix[mid * H]) * two_b <= g) la = mid; else lz = mid;
  }
  const int32_t c0 = prefix[la * H];
  const int64_t C2 = 2 * int64_t(prefix[(la + 1) * H] - c0);   // units per batch entry of the layer
  const int64_t r = g - int64_t(c0) * two_b;
  const int32_t rem = int32_t(r % C2);
  const int32_t c = c0 + (rem >> 1);
  int lo = la * H, hi = (la + 1) * H;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= c) lo = mid; else hi = mid;
  }
  uint32_t m = masks[lo] & cls;
  for (int32_t j = c - prefix[lo]; j > 0; --j) m &= m - 1;   // drop the j lowest kept scales
  QBlock q;
  q.s = __ffs(m) - 1;
  q.l = p.l0 + la;
  q.h = lo - la * H;
  q.b = int(r / C2);
  q.t = rem & 1;
  return q;
}

// Per-channel maximum of |x| over 8 bf16 channels, as magnitude bits.
__device__ __forceinline__ void absmax8(uint32_t (&acc)[4], const uint4& x) {
  acc[0] = __vmaxu2(acc[0], x.x & 0x7FFF7FFFu);
  acc[1] = __vmaxu2(acc[1], x.y & 0x7FFF7FFFu);
  acc[2] = __vmaxu2(acc[2], x.z & 0x7FFF7FFFu);
  acc[3] = __vmaxu2(acc[3], x.w & 0x7FFF7FFFu);
}

// Channel scale: 8-bit codes sc = a / 127 (IEEE); 4-bit codes sc = bf16(a / 7)
// and 3-bit codes sc = bf16(a / 3) (IEEE division rounded to bf16, the value the
// scale table stores);
// rc = RN(1 / sc) when the product path is usable (2^-100 <= sc <= 2^100),
// else 0 (always divide).
struct QScale {
  float sc, rc;
};

__device__ __forceinline__ float round_to_bf16(float x) { return __uint_as_float(pack_bf16x2(x, 0.f) << 16); }

template <int BITS>
__device__ __forceinline__ QScale make_qscale(float a) {
  QScale q;
  q.sc = BITS == 8 ? a / 127.f : round_to_bf16(a / (BITS == 4 ? 7.f : 3.f));
  q.rc = (q.sc >= 0x1p-100f && q.sc <= 0x1p100f) ? __frcp_rn(q.sc) : 0.f;
  return q;
}

// Codes of 8 channels: rint(x / sc) with x / sc the IEEE quotient, clamped to
// [-127, 127].  |x| <= a and sc = RN(a / 127) give |x / sc| <= 127 (1 + 2^-24),
// so the clamp never binds for finite inputs and is left out.  The product
// t = x * rc (rc = RN(1 / sc)) differs from the quotient by at most
// |t| * 1.5 * 2^-23 (two roundings of relative 2^-24, plus the quotient's own
// half ulp), so rint(t) = rint(quotient) unless t lies within that distance of
// a half-integer.  Elements whose t lies within 2^-13 of one (a band that
// contains every |t| * 2^-20 distance, since |t| <= 127 (1 + 2^-23); ties
// x = a / 2 are common in bf16 data) take the exact division instead.  The
// product and rounding steps run as packed f32x2 pairs.
__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Adding kRound = 1.5 * 2^23 rounds a float of magnitude below 2^22 to an
// integer (round to nearest, ties to even: the sum's ulp is 1), and the sum's
// low byte is then that integer's two's-complement byte.
constexpr float kRound = 12582912.0f;
// |t| <= 127 (1 + 2^-23) gives |t| * 2^-20 < 2^-13, so every element whose
// product may round differently from the quotient has |t - rint(t)| above
// this band.
constexpr float kTieBand = 0.5f - 0x1p-13f;

__device__ __forceinline__ uint32_t pack4_low_bytes(float y0, float y1, float y2, float y3) {
  return __byte_perm(__byte_perm(__float_as_uint(y0), __float_as_uint(y1), 0x0040),
                     __byte_perm(__float_as_uint(y2), __float_as_uint(y3), 0x0040), 0x5410);
}

// y[j] = kRound + rint(x_j / sc_j) for the 8 channels of one 16-byte vector.
// With 8-bit codes |x / sc| <= 127 (1 + 2^-24); with 4-bit codes sc = bf16(a / 7)
// >= (a / 7)(1 - 2^-8), so |x / sc| < 7.03, and with 3-bit codes |x / sc| < 3.02:
// rint never leaves [-127, 127] / [-7, 7] / [-3, 3] and no clamp is needed.
__device__ __forceinline__ void code_sums8(const uint4& x, const float (&sc)[8], const float (&rc)[8], bool force,
                                           float (&y)[8]) {
  const float v[8] = {lo_bf16(x.x), hi_bf16(x.x), lo_bf16(x.y), hi_bf16(x.y),
                      lo_bf16(x.z), hi_bf16(x.z), lo_bf16(x.w), hi_bf16(x.w)};
  float t[8], r[8], e[8];
#pragma unroll
  for (int j = 0; j < 8; j += 2) {
    ffma2(t[j], t[j + 1], v[j], v[j + 1], rc[j], rc[j + 1], 0.f, 0.f);           // t = RN(x * rc)
    fadd2(y[j], y[j + 1], t[j], t[j + 1], kRound, kRound);                      // kRound + rint(t)
    fadd2(r[j], r[j + 1], y[j], y[j + 1], -kRound, -kRound);                    // rint(t), exact
    ffma2(e[j], e[j + 1], r[j], r[j + 1], -1.f, -1.f, t[j], t[j + 1]);           // t - rint(t), exact
  }
  const float emax = fmaxf(fmaxf(fmaxf(fabsf(e[0]), fabsf(e[1])), fmaxf(fabsf(e[2]), fabsf(e[3]))),
                           fmaxf(fmaxf(fabsf(e[4]), fabsf(e[5])), fmaxf(fabsf(e[6]), fabsf(e[7]))));
  if (force || emax > kTieBand) {   // rare: decide the flagged elements by the exact quotient
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (force || fabsf(e[j]) > kTieBand) y[j] = __fadd_rn(sc[j] == 0.f ? 0.f : __fdiv_rn(v[j], sc[j]), kRound);
  }
}

// 8-bit codes: one byte per channel, in channel order.
__device__ __forceinline__ uint2 codes8(const uint4& x, const float (&sc)[8], const float (&rc)[8], bool force) {
  float y[8];
  code_sums8(x, sc, rc, force, y);
  uint2 o;
  o.x = pack4_low_bytes(y[0], y[1], y[2], y[3]);
  o.y = pack4_low_bytes(y[4], y[5], y[6], y[7]);
  return o;
}

// 4-bit codes: nibble = code + 8; channels 0, 2, 4, 6 in nibbles 0-3 and 1, 3,
// 5, 7 in nibbles 4-7 of one word (the low bits of kRound + code + 8 are the
// nibble).  That order lets a consumer form bf16 pairs of adjacent channels
// with one mask per pair.
__device__ __forceinline__ uint32_t codes4x8(const uint4& x, const float (&sc)[8], const float (&rc)[8], bool force) {
  float y[8];
  code_sums8(x, sc, rc, force, y);
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    w |= ((__float_as_uint(y[2 * j]) + 8u) & 0xFu) << (4 * j);
    w |= ((__float_as_uint(y[2 * j + 1]) + 8u) & 0xFu) << (16 + 4 * j);
  }
  return w;
}

// 3-bit codes: field = code + 4 at bits 3j of a 24-bit group (8 channels, 3
// bytes, little-endian); the low bits of kRound + code + 4 are the field.
__device__ __forceinline__ uint32_t codes3x8(const uint4& x, const float (&sc)[8], const float (&rc)[8], bool force) {
  float y[8];
  code_sums8(x, sc, rc, force, y);
  uint32_t w = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) w |= ((__float_as_uint(y[j]) + 4u) & 0x7u) << (3 * j);
  return w;
}

__device__ __forceinline__ void store3(uint8_t* p, uint32_t w) {
  p[0] = uint8_t(w);
  p[1] = uint8_t(w >> 8);
  p[2] = uint8_t(w >> 16);
}

// BITS = 8: kq / vq int8 codes (one byte per element), ka / va fp32 absmax.
// BITS = 4: kq / vq packed nibbles (one 32-bit word per 8 elements), ka / va
// bf16 bits (uint16) of the scale bf16(a / 7).
// BITS = 3: kq / vq 24-bit groups (3 bytes per 8 elements), ka / va bf16 bits
// of the scale bf16(a / 3).
template <int BITS>
__global__ void __cluster_dims__(kQuantCluster, 1, 1) __launch_bounds__(kQuantThreads, 5) quant_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, QuantParams p, const uint8_t* __restrict__ keep,
    const int32_t* __restrict__ head_off, const int32_t* __restrict__ seg_off, const int64_t* __restrict__ layer_base,
    void* __restrict__ kq, void* __restrict__ vq, void* __restrict__ ka, void* __restrict__ va) {
  __shared__ int32_t big_prefix[kQuantGroupLH + 1];
  __shared__ int32_t small_prefix[kQuantGroupLH + 1];
  __shared__ uint32_t keep_mask[kQuantGroupLH];
  __shared__ int32_t warp_tot[kQuantThreads / 32];
  __shared__ __align__(16) uint32_t red[kQuantThreads * 4];
  __shared__ uint32_t part[2][kQuantMaxD / 2];   // read by the other CTAs of the cluster
  __shared__ uint32_t fin[kQuantMaxD / 2];
  __shared__ __align__(16) float fin_sc[kQuantMaxD];   // a / 127 per channel
  __shared__ __align__(16) float fin_rc[kQuantMaxD];   // RN(1 / (a / 127)), or 0: divide

  const int S = p.sc.S, H = p.H, D = p.D, B = p.B;
  const int nlh = p.nl * H;
  const int lh0 = p.l0 * H;
  for (int i = threadIdx.x; i < nlh; i += kQuantThreads) {
    const uint8_t* kp = keep + int64_t(lh0 + i) * S;
    uint32_t m = 0;
    for (int s = 0; s < S; ++s)
      if (kp[s]) m |= 1u << s;
    keep_mask[i] = m;
    big_prefix[i] = __popc(m & p.big_mask);
    small_prefix[i] = __popc(m & ~p.big_mask);
  }
  __syncthreads();
  block_exclusive_scan<kQuantThreads, kQuantGroupLH>(big_prefix, nlh, warp_tot);
  block_exclusive_scan<kQuantThreads, kQuantGroupLH>(small_prefix, nlh, warp_tot);

  const int64_t n_big = int64_t(big_prefix[nlh]) * 2 * B;
  const int64_t n_small = int64_t(small_prefix[nlh]) * 2 * B;
  const int64_t n_units = n_big + (n_small + kQuantCluster - 1) / kQuantCluster;
  const uint32_t rank = cluster_ctarank();
  const int cv_n = D / 8;                         // 16-byte vectors per row
  const int nrg = kQuantThreads / cv_n;           // row groups
  const bool active = threadIdx.x < nrg * cv_n;
  const int cv = threadIdx.x % cv_n;
  const int rg = threadIdx.x / cv_n;
  const int dw = D / 2;                           // channel-pair words per row
  int parity = 0;

  // Units are taken cluster-wide: big blocks first, then packs of kQuantCluster
  // small blocks (one per CTA).  Every CTA of a cluster runs the same
  // iterations, so the cluster barriers below match up.
  for (int64_t u = cluster_id_x(); u < n_units; u += cluster_count_x()) {
    const bool big = u < n_big;
    const int64_t g = big ? u : (u - n_big) * kQuantCluster + rank;
    const bool have = big || g < n_small;
    QBlock q{0, 0, 0, 0, 0};
    int32_t r_lo = 0, r_hi = 0;
    if (have) {
      q = big ? decode_block(g, big_prefix, keep_mask, p.big_mask, p)
              : decode_block(g, small_prefix, keep_mask, ~p.big_mask, p);
      const int32_t n = p.sc.n[q.s];
      if (big) {
        const int32_t per = (n + kQuantCluster - 1) / kQuantCluster;
        r_lo = min(n, int32_t(rank) * per);
        r_hi = min(n, r_lo + per);
      } else {
        r_hi = n;
      }
    }
    // this CTA's first row of the block; rows below are 32-bit offsets (a block has at most 2^31 / D rows)
    const uint4* src = (q.t ? v : k) +
                       (int64_t(q.l) * p.layer_stride + ((int64_t(q.b) * H + q.h) * p.sc.T + p.sc.off[q.s]) * D) / 8 +
                       int64_t(r_lo) * cv_n + cv;
    const int32_t nr = r_hi - r_lo;
    // 1. channel maxima of this CTA's rows (normal caching: pass 2 re-reads them)
    uint32_t acc[4] = {0u, 0u, 0u, 0u};
    if (active) {
      int32_t r = rg;
      for (; r + 7 * nrg < nr; r += 8 * nrg) {
        uint4 x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = __ldg(src + (r + e * nrg) * cv_n);
#pragma unroll
        for (int e = 0; e < 8; ++e) absmax8(acc, x[e]);
      }
      for (; r < nr; r += nrg) absmax8(acc, __ldg(src + r * cv_n));
      *reinterpret_cast<uint4*>(&red[threadIdx.x * 4]) = make_uint4(acc[0], acc[1], acc[2], acc[3]);
    }
    __syncthreads();
    // channel pairs x = threadIdx.x, threadIdx.x + kQuantThreads, ... (below dw)
    for (int x = threadIdx.x; x < dw; x += kQuantThreads) {
      uint32_t w = 0;
      for (int e = 0; e < nrg; ++e) w = __vmaxu2(w, red[e * dw + x]);
      if (big) part[parity][x] = w; else fin[x] = w;
    }
    if (big) {
      cluster_sync_all();
      for (int x = threadIdx.x; x < dw; x += kQuantThreads) {
        const uint32_t a = smem_u32(&part[parity][x]);
        uint32_t w = 0;
        for (uint32_t c = 0; c < kQuantCluster; ++c)
          w = __vmaxu2(w, __float_as_uint(ld_shared_cluster_f32(map_shared_rank(a, c))));
        fin[x] = w;
      }
      parity ^= 1;   // the next big unit writes the other buffer while peers may still read this one
    }
    for (int x = threadIdx.x; x < dw; x += kQuantThreads) {   // the pair's scales, once per unit
      const uint32_t w = fin[x];
      const QScale q0 = make_qscale<BITS>(lo_bf16(w)), q1 = make_qscale<BITS>(hi_bf16(w));
      fin_sc[2 * x] = q0.sc;
      fin_sc[2 * x + 1] = q1.sc;
      fin_rc[2 * x] = q0.rc;
      fin_rc[2 * x + 1] = q1.rc;
    }
    __syncthreads();
    if (!have) continue;
    // 2. codes of this CTA's rows
    if (active && nr > 0) {
      float sc[8], rc[8];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float4 a = *reinterpret_cast<const float4*>(&fin_sc[cv * 8 + 4 * e]);
        const float4 b = *reinterpret_cast<const float4*>(&fin_rc[cv * 8 + 4 * e]);
        sc[4 * e] = a.x; sc[4 * e + 1] = a.y; sc[4 * e + 2] = a.z; sc[4 * e + 3] = a.w;
        rc[4 * e] = b.x; rc[4 * e + 1] = b.y; rc[4 * e + 2] = b.z; rc[4 * e + 3] = b.w;
      }
      bool force = false;   // a channel whose scale is non-zero but has no usable reciprocal
#pragma unroll
      for (int j = 0; j < 8; ++j) force |= sc[j] != 0.f && rc[j] == 0.f;
      const int64_t R_l = (layer_base[q.l + 1] - layer_base[q.l]) / (int64_t(B) * D);
      const int64_t row0 =
          int64_t(q.b) * R_l + head_off[q.l * H + q.h] + seg_off[(int64_t(q.l) * H + q.h) * S + q.s];
      // element index of this CTA's first row; 8 elements per 8-byte (int8) or 4-byte (int4) store
      const int64_t e_first = layer_base[q.l] + (row0 + r_lo) * D;
      int32_t r = rg;
      if (BITS == 3) {
        uint8_t* dst = static_cast<uint8_t*>(q.t ? vq : kq) + (e_first / 8) * 3 + cv * 3;
        for (; r + 3 * nrg < nr; r += 4 * nrg) {
          uint4 x[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) x[e] = __ldcs(src + (r + e * nrg) * cv_n);
#pragma unroll
          for (int e = 0; e < 4; ++e) store3(dst + int64_t(r + e * nrg) * cv_n * 3, codes3x8(x[e], sc, rc, force));
        }
        for (; r < nr; r += nrg) store3(dst + int64_t(r) * cv_n * 3, codes3x8(__ldcs(src + r * cv_n), sc, rc, force));
      } else if (BITS == 8) {
        uint2* dst = reinterpret_cast<uint2*>(static_cast<int8_t*>(q.t ? vq : kq) + e_first) + cv;
        for (; r + 3 * nrg < nr; r += 4 * nrg) {
          uint4 x[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) x[e] = __ldcs(src + (r + e * nrg) * cv_n);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[(r + e * nrg) * cv_n] = codes8(x[e], sc, rc, force);
        }
        for (; r < nr; r += nrg) dst[r * cv_n] = codes8(__ldcs(src + r * cv_n), sc, rc, force);
      } else {
        uint32_t* dst = static_cast<uint32_t*>(q.t ? vq : kq) + e_first / 8 + cv;
        for (; r + 3 * nrg < nr; r += 4 * nrg) {
          uint4 x[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) x[e] = __ldcs(src + (r + e * nrg) * cv_n);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[(r + e * nrg) * cv_n] = codes4x8(x[e], sc, rc, force);
        }
        for (; r < nr; r += nrg) dst[r * cv_n] = codes4x8(__ldcs(src + r * cv_n), sc, rc, force);
      }
    }
    // the block's absmax entries: once per block
    if (!big || rank == 0) {
      const int64_t t0 = ((((int64_t(q.l) * B + q.b) * H + q.h) * S) + q.s) * D;
      for (int c = threadIdx.x; c < D; c += kQuantThreads) {
        const uint32_t w = fin[c >> 1];
        const float a = (c & 1) ? hi_bf16(w) : lo_bf16(w);
        if (BITS == 8) static_cast<float*>(q.t ? va : ka)[t0 + c] = a;
        else static_cast<uint16_t*>(q.t ? va : ka)[t0 + c] = uint16_t(__float_as_uint(make_qscale<BITS>(a).sc) >> 16);
      }
    }
  }
  cluster_sync_all();   // no CTA leaves while a peer may still read its partial maxima
}

// Dequantisation of one layer.  Unit = (batch, head, kept scale, chunk of at
// most kDeqRows rows), in that (memory) order; each thread keeps the scales of
// its 8 channels for the unit and streams rows, four at a time: 8-byte code
// loads, 16-byte bf16 stores (normal caching: the attention that follows reads
// them).
constexpr int kDeqRows = 128;
constexpr int kDeqThreads = 256;
constexpr int kDeqMaxH = 4096;

struct DequantParams {
  ScaleTable sc;
  int B, H, D;
  int64_t R;               // rows per batch entry of the layer
};

// BITS = 8: codes are uint2 per 8 elements, tables fp32 absmax (scale a / 127).
// BITS = 4: codes are one uint32 word per 8 elements, tables bf16 scale bits.
// BITS = 3: codes are 3 bytes per 8 elements (a 24-bit group), tables bf16 scale bits.
template <int BITS>
__global__ void __launch_bounds__(kDeqThreads, 3) dequant_kernel(const void* __restrict__ kq_,
                                                              const void* __restrict__ vq_,
                                                              const void* __restrict__ ka_,
                                                              const void* __restrict__ va_, DequantParams p,
                                                              const int32_t* __restrict__ head_off,
                                                              const int32_t* __restrict__ seg_off,
                                                              uint4* __restrict__ kc, uint4* __restrict__ vc) {
  using CodeVec = typename std::conditional<BITS == 8, uint2, uint32_t>::type;
  // code group e (8 elements) of a code buffer
  auto load_codes = [](const void* base, int64_t e) -> CodeVec {
    if constexpr (BITS == 3) {
      const uint8_t* b = static_cast<const uint8_t*>(base) + e * 3;
      return uint32_t(__ldcs(b)) | (uint32_t(__ldcs(b + 1)) << 8) | (uint32_t(__ldcs(b + 2)) << 16);
    } else {
      return __ldcs(static_cast<const CodeVec*>(base) + e);
    }
  };
  __shared__ int32_t prefix[kDeqMaxH + 1];
  __shared__ uint32_t masks[kDeqMaxH];
  __shared__ int32_t warp_tot[kDeqThreads / 32];
  const int S = p.sc.S, H = p.H, D = p.D, B = p.B;
  for (int h = threadIdx.x; h < H; h += kDeqThreads) {
    uint32_t m = 0;
    int32_t c = 0;
    for (int s = 0; s < S; ++s)
      if (seg_off[h * S + s] >= 0) {
        m |= 1u << s;
        c += (p.sc.n[s] + kDeqRows - 1) / kDeqRows;
      }
    masks[h] = m;
    prefix[h] = c;
  }
  __syncthreads();
  block_exclusive_scan<kDeqThreads, kDeqMaxH>(prefix, H, warp_tot);
  const int32_t C = prefix[H];                 // chunks per batch entry of the layer
  const int64_t units = int64_t(C) * B;
  const int cv_n = D / 8;
  const int nrg = kDeqThreads / cv_n;
  if (threadIdx.x >= nrg * cv_n) return;   // no block-wide barrier follows
  const int cv = threadIdx.x % cv_n;
  const int rg = threadIdx.x / cv_n;
  // Code byte i of w as a float, on the integer and FMA pipes: with the sign
  // bit flipped the byte is k + 128, placed as the low mantissa byte of
  // 1.5 * 2^23 (bits 0x4B400000) it reads 1.5 * 2^23 + k + 128, and one exact
  // subtraction leaves k.
  auto expand8 = [](uint2 w, const float (&sc)[8]) {
    const uint2 wf = make_uint2(w.x ^ 0x80808080u, w.y ^ 0x80808080u);
    auto x = [](uint32_t u, int i) {
      return __fsub_rn(__uint_as_float(__byte_perm(u, 0x4B400000u, 0x7640u | uint32_t(i))), 12583040.0f);
    };
    uint4 o;
    o.x = pack_bf16x2(__fmul_rn(x(wf.x, 0), sc[0]), __fmul_rn(x(wf.x, 1), sc[1]));
    o.y = pack_bf16x2(__fmul_rn(x(wf.x, 2), sc[2]), __fmul_rn(x(wf.x, 3), sc[3]));
    o.z = pack_bf16x2(__fmul_rn(x(wf.y, 0), sc[4]), __fmul_rn(x(wf.y, 1), sc[5]));
    o.w = pack_bf16x2(__fmul_rn(x(wf.y, 2), sc[6]), __fmul_rn(x(wf.y, 3), sc[7]));
    return o;
  };
  // A nibble n (code + 8) placed in the low mantissa bits of 1.5 * 2^23 reads
  // 1.5 * 2^23 + n; subtracting 1.5 * 2^23 + 8 leaves the code exactly.  The
  // product code * sc has at most 11 significant bits, so it is exact in fp32
  // and the bf16 conversion rounds it once.
  auto expand4 = [](uint32_t w, const float (&sc)[8]) {
    auto x = [](uint32_t u, int shift) {
      return __fsub_rn(__uint_as_float(0x4B400000u | ((u >> shift) & 0xFu)), 12582920.0f);
    };
    uint4 o;
    o.x = pack_bf16x2(__fmul_rn(x(w, 0), sc[0]), __fmul_rn(x(w, 16), sc[1]));
    o.y = pack_bf16x2(__fmul_rn(x(w, 4), sc[2]), __fmul_rn(x(w, 20), sc[3]));
    o.z = pack_bf16x2(__fmul_rn(x(w, 8), sc[4]), __fmul_rn(x(w, 24), sc[5]));
    o.w = pack_bf16x2(__fmul_rn(x(w, 12), sc[6]), __fmul_rn(x(w, 28), sc[7]));
    return o;
  };
  // A 3-bit field f (code + 4) reads 1.5 * 2^23 + f in the same way; the
  // product code * sc has at most 10 significant bits.
  auto expand3 = [](uint32_t w, const float (&sc)[8]) {
    auto x = [](uint32_t u, int shift) {
      return __fsub_rn(__uint_as_float(0x4B400000u | ((u >> shift) & 0x7u)), 12582916.0f);
    };
    uint4 o;
    o.x = pack_bf16x2(__fmul_rn(x(w, 0), sc[0]), __fmul_rn(x(w, 3), sc[1]));
    o.y = pack_bf16x2(__fmul_rn(x(w, 6), sc[2]), __fmul_rn(x(w, 9), sc[3]));
    o.z = pack_bf16x2(__fmul_rn(x(w, 12), sc[4]), __fmul_rn(x(w, 15), sc[5]));
    o.w = pack_bf16x2(__fmul_rn(x(w, 18), sc[6]), __fmul_rn(x(w, 21), sc[7]));
    return o;
  };
  auto expand = [&](CodeVec w, const float (&sc)[8]) {
    if constexpr (BITS == 8) return expand8(w, sc);
    else if constexpr (BITS == 4) return expand4(w, sc);
    else return expand3(w, sc);
  };
  // units in memory order (batch, head, kept chunk)
  for (int64_t g = blockIdx.x; g < units; g += gridDim.x) {
    const int b = int(g / C);
    const int32_t c = int32_t(g % C);
    int lo = 0, hi = H;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= c) lo = mid; else hi = mid;
    }
    const int h = lo;
    int32_t j = c - prefix[h];
    const uint32_t m = masks[h];
    int s = 0;
    for (; s < S; ++s)
      if (m >> s & 1u) {
        const int32_t ch = (p.sc.n[s] + kDeqRows - 1) / kDeqRows;
        if (j < ch) break;
        j -= ch;
      }
    const int32_t r0 = j * kDeqRows;
    const int32_t nrows = min(kDeqRows, p.sc.n[s] - r0);
    const int64_t row0 = int64_t(b) * p.R + head_off[h] + seg_off[h * S + s] + r0;
    const int64_t arow = ((int64_t(b) * H + h) * S + s) * D + cv * 8;
    float sk[8], sv[8];
    if constexpr (BITS == 8) {
      const float* ka = static_cast<const float*>(ka_);
      const float* va = static_cast<const float*>(va_);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float4 a = *reinterpret_cast<const float4*>(ka + arow + 4 * e);
        const float4 bq = *reinterpret_cast<const float4*>(va + arow + 4 * e);
        sk[4 * e] = a.x / 127.f; sk[4 * e + 1] = a.y / 127.f; sk[4 * e + 2] = a.z / 127.f; sk[4 * e + 3] = a.w / 127.f;
        sv[4 * e] = bq.x / 127.f; sv[4 * e + 1] = bq.y / 127.f; sv[4 * e + 2] = bq.z / 127.f; sv[4 * e + 3] = bq.w / 127.f;
      }
    } else {
      const uint4 a = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(ka_) + arow);
      const uint4 bq = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(va_) + arow);
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        sk[2 * e] = lo_bf16(wa[e]); sk[2 * e + 1] = hi_bf16(wa[e]);
        sv[2 * e] = lo_bf16(wb[e]); sv[2 * e + 1] = hi_bf16(wb[e]);
      }
    }
    const int64_t e0 = row0 * cv_n + cv;
    int32_t r = rg;
    for (; r + 3 * nrg < nrows; r += 4 * nrg) {     // 4 rows' loads in flight, then the stores
      CodeVec ck[4], cw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        ck[u] = load_codes(kq_, e0 + int64_t(r + u * nrg) * cv_n);
        cw[u] = load_codes(vq_, e0 + int64_t(r + u * nrg) * cv_n);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        kc[e0 + int64_t(r + u * nrg) * cv_n] = expand(ck[u], sk);
        vc[e0 + int64_t(r + u * nrg) * cv_n] = expand(cw[u], sv);
      }
    }
    for (; r < nrows; r += nrg) {
      const int64_t e = e0 + int64_t(r) * cv_n;
      const CodeVec ck = load_codes(kq_, e);
      const CodeVec cw = load_codes(vq_, e);
      kc[e] = expand(ck, sk);
      vc[e] = expand(cw, sv);
    }
  }
}

}  // namespace vark

using namespace vark;

template <int BITS>
static int quantize_kv(const uint16_t* k, const uint16_t* v, int64_t layer_stride, int L, int B, int H, int S, int D,
                       const int32_t* sides, const uint8_t* keep, const int32_t* head_off, const int32_t* seg_off,
                       const int64_t* layer_base, void* kq, void* vq, void* k_tab, void* v_tab, void* stream) {
  if (!k || !v || !keep || !head_off || !seg_off || !layer_base || !kq || !vq || !k_tab || !v_tab)
    return VARK_E_ARG;
  QuantParams q;
  int rc = make_scale_table(S, sides, &q.sc);
  if (rc) return rc;
  if (L < 1 || H < 1 || B < 1 || D < 8 || D % 8 != 0 || D > kQuantMaxD) return VARK_E_SHAPE;
  if (H > kQuantGroupLH) return VARK_E_SHAPE;
  for (int s = 0; s < S; ++s)   // rows of a block are addressed with 32-bit vector offsets
    if (int64_t(q.sc.n[s]) * (D / 8) >= INT32_MAX) return VARK_E_SHAPE;
  if (layer_stride < int64_t(B) * H * q.sc.T * D) return VARK_E_ARG;
  if (layer_stride % 8 != 0) return VARK_E_ALIGN;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kq) || !aligned16(vq) || !aligned16(k_tab) || !aligned16(v_tab))
    return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t ntab = int64_t(L) * B * H * S * D * (BITS == 8 ? 4 : 2);
  if (cudaMemsetAsync(k_tab, 0, size_t(ntab), st) != cudaSuccess ||
      cudaMemsetAsync(v_tab, 0, size_t(ntab), st) != cudaSuccess)
    return VARK_E_CUDA;
  q.L = L; q.B = B; q.H = H; q.D = D; q.layer_stride = layer_stride;
  q.big_mask = 0;
  for (int s = 0; s < S; ++s)
    if (q.sc.n[s] > kSmallRows) q.big_mask |= 1u << s;
  // as many clusters as can be resident at once (the unit loop is static)
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  int clusters = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nsm * 4 / kQuantCluster * kQuantCluster);
  cfg.blockDim = dim3(kQuantThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  if (cudaOccupancyMaxActiveClusters(&clusters, quant_kernel<BITS>, &cfg) != cudaSuccess || clusters < 1) {
    cudaGetLastError();
    clusters = std::max(1, nsm / kQuantCluster);
  }
  const int layers_per_group = std::max(1, kQuantGroupLH / H);
  for (int l0 = 0; l0 < L; l0 += layers_per_group) {
    q.l0 = l0;
    q.nl = std::min(layers_per_group, L - l0);
    quant_kernel<BITS><<<clusters * kQuantCluster, kQuantThreads, 0, st>>>(
        reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), q, keep, head_off, seg_off, layer_base,
        kq, vq, k_tab, v_tab);
    if (cudaGetLastError() != cudaSuccess) return VARK_E_CUDA;
  }
  return VARK_OK;
}

template <int BITS>
static int dequantize_layer(const void* kq, const void* vq, const void* k_tab, const void* v_tab, int64_t kc_rows,
                            int B, int H, int S, int D, const int32_t* sides, const int32_t* head_off,
                            const int32_t* seg_off, uint16_t* kc, uint16_t* vc, void* stream) {
  if (!kq || !vq || !k_tab || !v_tab || !head_off || !seg_off || !kc || !vc) return VARK_E_ARG;
  DequantParams p;
  int rc = make_scale_table(S, sides, &p.sc);
  if (rc) return rc;
  if (B < 1 || H < 1 || H > kDeqMaxH || D < 8 || D % 8 != 0 || D > 512 || kc_rows < 0 || kc_rows % B != 0)
    return VARK_E_SHAPE;
  const uintptr_t code_align = BITS == 8 ? 7 : BITS == 4 ? 3 : 0;
  if (!aligned16(k_tab) || !aligned16(v_tab) || (reinterpret_cast<uintptr_t>(kq) & code_align) ||
      (reinterpret_cast<uintptr_t>(vq) & code_align) || !aligned16(kc) || !aligned16(vc))
    return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  if (kc_rows == 0) return VARK_OK;
  p.B = B; p.H = H; p.D = D; p.R = kc_rows / B;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  dequant_kernel<BITS><<<nsm * 3, kDeqThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      kq, vq, k_tab, v_tab, p, head_off, seg_off, reinterpret_cast<uint4*>(kc), reinterpret_cast<uint4*>(vc));
  return cudaGetLastError() == cudaSuccess ? VARK_OK : VARK_E_CUDA;
}

extern "C" int vark_quantize_kv_int8(const uint16_t* k, const uint16_t* v, int64_t layer_stride, int L, int B, int H,
                                     int S, int D, const int32_t* sides, const uint8_t* keep,
                                     const int32_t* head_off, const int32_t* seg_off, const int64_t* layer_base,
                                     int8_t* kq, int8_t* vq, float* k_absmax, float* v_absmax, void* stream) {
  return quantize_kv<8>(k, v, layer_stride, L, B, H, S, D, sides, keep, head_off, seg_off, layer_base, kq, vq,
                        k_absmax, v_absmax, stream);
}

extern "C" int vark_quantize_kv_int4(const uint16_t* k, const uint16_t* v, int64_t layer_stride, int L, int B, int H,
                                     int S, int D, const int32_t* sides, const uint8_t* keep,
                                     const int32_t* head_off, const int32_t* seg_off, const int64_t* layer_base,
                                     uint8_t* kq, uint8_t* vq, uint16_t* k_scale, uint16_t* v_scale, void* stream) {
  return quantize_kv<4>(k, v, layer_stride, L, B, H, S, D, sides, keep, head_off, seg_off, layer_base, kq, vq,
                        k_scale, v_scale, stream);
}

extern "C" int vark_quantize_kv_int3(const uint16_t* k, const uint16_t* v, int64_t layer_stride, int L, int B, int H,
                                     int S, int D, const int32_t* sides, const uint8_t* keep,
                                     const int32_t* head_off, const int32_t* seg_off, const int64_t* layer_base,
                                     uint8_t* kq, uint8_t* vq, uint16_t* k_scale, uint16_t* v_scale, void* stream) {
  return quantize_kv<3>(k, v, layer_stride, L, B, H, S, D, sides, keep, head_off, seg_off, layer_base, kq, vq,
                        k_scale, v_scale, stream);
}

extern "C" int vark_dequantize_layer_int8(const int8_t* kq, const int8_t* vq, const float* k_absmax,
                                          const float* v_absmax, int64_t kc_rows, int B, int H, int S, int D,
                                          const int32_t* sides, const int32_t* head_off, const int32_t* seg_off,
                                          uint16_t* kc, uint16_t* vc, void* stream) {
  return dequantize_layer<8>(kq, vq, k_absmax, v_absmax, kc_rows, B, H, S, D, sides, head_off, seg_off, kc, vc,
                             stream);
}

extern "C" int vark_dequantize_layer_int4(const uint8_t* kq, const uint8_t* vq, const uint16_t* k_scale,
                                          const uint16_t* v_scale, int64_t kc_rows, int B, int H, int S, int D,
                                          const int32_t* sides, const int32_t* head_off, const int32_t* seg_off,
                                          uint16_t* kc, uint16_t* vc, void* stream) {
  return dequantize_layer<4>(kq, vq, k_scale, v_scale, kc_rows, B, H, S, D, sides, head_off, seg_off, kc, vc,
                             stream);
}

extern "C" int vark_dequantize_layer_int3(const uint8_t* kq, const uint8_t* vq, const uint16_t* k_scale,
                                          const uint16_t* v_scale, int64_t kc_rows, int B, int H, int S, int D,
                                          const int32_t* sides, const int32_t* head_off, const int32_t* seg_off,
                                          uint16_t* kc, uint16_t* vc, void* stream) {
  return dequantize_layer<3>(kq, vq, k_scale, v_scale, kc_rows, B, H, S, D, sides, head_off, seg_off, kc, vc,
                             stream);
}
