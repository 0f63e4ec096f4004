// Offset tables and cache compaction: apply a static keep[layer][head][scale]
// schedule by gathering the retained scale blocks of every (layer, batch,
// head) into the per-head ragged layout documented in vark.h.
// [HeatKV] project page, Method step 5: the static schedule is applied while
// scales are generated; the Abstract: allocation is head-specific.
//
// Compaction is a pure HBM stream (every retained byte read once and written
// once, dropped bytes never touched).  Work unit = (layer, head, kept chunk of
// <= kChunkRows rows of one scale, batch); one persistent grid walks the units.
// Each CTA first builds, in shared memory, the prefix of kept chunks over
// (layer, head) for its layer group, so a unit is found by one binary search
// and a walk over at most S scales.  Copies are 16-byte vectors, coalesced,
// with several loads in flight per thread before the stores.
#include <algorithm>

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
constexpr int kChunkRows = 64;
constexpr int kCompactThreads = 256;
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

__global__ void __launch_bounds__(kCompactThreads) compact_kernel(
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
  // 2. in-place exclusive scan: each thread owns a contiguous segment
  constexpr int kPer = (kMaxGroupLH + kCompactThreads - 1) / kCompactThreads;
  const int seg0 = threadIdx.x * kPer;
  int32_t my_total = 0;
  for (int u = 0; u < kPer; ++u)
    if (seg0 + u < nlh) my_total += chunk_prefix[seg0 + u];
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
  for (int w = 0; w < kCompactThreads / 32; ++w) {
    if (w < warp) warp_base += warp_tot[w];
    grand += warp_tot[w];
  }
  int32_t run = warp_base + incl - my_total;
  for (int u = 0; u < kPer; ++u) {
    if (seg0 + u < nlh) {
      const int32_t c = chunk_prefix[seg0 + u];
      chunk_prefix[seg0 + u] = run;
      run += c;
    }
  }
  if (threadIdx.x == 0) chunk_prefix[nlh] = grand;
  __syncthreads();

  const int64_t units = int64_t(grand) * p.B;
  const int vec_per_row = p.D / 8;  // 16-byte vectors per row

  for (int64_t g = blockIdx.x; g < units; g += gridDim.x) {
    const int b = int(g % p.B);
    const int32_t c = int32_t(g / p.B);
    // (layer, head) with chunk_prefix[i] <= c < chunk_prefix[i+1]
    int lo = 0, hi = nlh;
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

    // 4 K + 4 V vectors in flight per thread, then the stores.
    for (int base = 0; base < nvec; base += 4 * kCompactThreads) {
      uint4 a[4], bq[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = base + u * kCompactThreads + threadIdx.x;
        if (e < nvec) {
          a[u] = __ldcs(k + src_v + e);
          bq[u] = __ldcs(v + src_v + e);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
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

namespace vark {

constexpr int kQuantThreads = 256;

struct QuantParams {
  CompactParams c;          // layout and unit walk (dense source)
  int mode;                 // 0: absmax pass, 1: quantise pass
  int64_t scale_stride_l;   // B*H*S*D
};

// One unit = (layer, head, kept chunk, batch) as in compact_kernel.  Every
// thread owns one channel-pair column of the chunk (D/2 columns) and strides
// over its rows.
__global__ void __launch_bounds__(kQuantThreads) quant_kernel(
    const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, QuantParams q, const uint8_t* __restrict__ keep,
    const int32_t* __restrict__ head_off, const int32_t* __restrict__ seg_off, const int64_t* __restrict__ layer_base,
    int8_t* __restrict__ kq, int8_t* __restrict__ vq, float* __restrict__ ka, float* __restrict__ va) {
  const CompactParams& p = q.c;
  __shared__ int32_t chunk_prefix[kMaxGroupLH + 1];
  __shared__ uint32_t keep_mask[kMaxGroupLH];
  __shared__ int32_t warp_tot[kQuantThreads / 32];
  const int S = p.sc.S;
  const int H = p.H;
  const int nlh = p.nl * H;
  const int lh0 = p.l0 * H;
  for (int i = threadIdx.x; i < nlh; i += kQuantThreads) {
    const uint8_t* kp = keep + int64_t(lh0 + i) * S;
    uint32_t m = 0;
    int32_t c = 0;
    for (int s = 0; s < S; ++s)
      if (kp[s] && p.chunks[s] > 0) {
        m |= 1u << s;
        c += p.chunks[s];
      }
    keep_mask[i] = m;
    chunk_prefix[i] = c;
  }
  __syncthreads();
  constexpr int kPer = (kMaxGroupLH + kQuantThreads - 1) / kQuantThreads;
  const int seg0 = threadIdx.x * kPer;
  int32_t my_total = 0;
  for (int u = 0; u < kPer; ++u)
    if (seg0 + u < nlh) my_total += chunk_prefix[seg0 + u];
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
  for (int w = 0; w < kQuantThreads / 32; ++w) {
    if (w < warp) warp_base += warp_tot[w];
    grand += warp_tot[w];
  }
  int32_t run = warp_base + incl - my_total;
  for (int u = 0; u < kPer; ++u)
    if (seg0 + u < nlh) {
      const int32_t c = chunk_prefix[seg0 + u];
      chunk_prefix[seg0 + u] = run;
      run += c;
    }
  if (threadIdx.x == 0) chunk_prefix[nlh] = grand;
  __syncthreads();

  const int64_t units = int64_t(grand) * p.B;
  const int cols = p.D / 2;                          // channel pairs
  const int col = threadIdx.x % cols;
  const int rstep = kQuantThreads / cols;
  const int rofs = threadIdx.x / cols;
  for (int64_t g = blockIdx.x; g < units; g += gridDim.x) {
    const int b = int(g % p.B);
    const int32_t c = int32_t(g / p.B);
    int lo = 0, hi = nlh;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (chunk_prefix[mid] <= c) lo = mid; else hi = mid;
    }
    const int i = lo;
    int32_t j = c - chunk_prefix[i];
    const uint32_t m = keep_mask[i];
    int s = 0;
    for (; s < S; ++s)
      if (m >> s & 1u) {
        if (j < p.chunks[s]) break;
        j -= p.chunks[s];
      }
    const int l = p.l0 + i / H;
    const int h = i % H;
    const int32_t r0 = j * kChunkRows;
    const int32_t nrows = min(kChunkRows, p.sc.n[s] - r0);
    const int64_t src_row0 = (int64_t(b) * H + h) * p.src_rows + p.src_off[s] + r0;
    const uint16_t* ks = k + int64_t(l) * p.layer_stride + src_row0 * p.D + 2 * col;
    const uint16_t* vs = v + int64_t(l) * p.layer_stride + src_row0 * p.D + 2 * col;
    float* kav = ka + int64_t(l) * q.scale_stride_l + ((int64_t(b) * H + h) * S + s) * p.D + 2 * col;
    float* vav = va + int64_t(l) * q.scale_stride_l + ((int64_t(b) * H + h) * S + s) * p.D + 2 * col;
    if (q.mode == 0) {
      float mk0 = 0.f, mk1 = 0.f, mv0 = 0.f, mv1 = 0.f;
      for (int r = rofs; r < nrows; r += rstep) {
        const uint32_t wk = *reinterpret_cast<const uint32_t*>(ks + int64_t(r) * p.D);
        const uint32_t wv = *reinterpret_cast<const uint32_t*>(vs + int64_t(r) * p.D);
        mk0 = fmaxf(mk0, fabsf(__uint_as_float(wk << 16)));
        mk1 = fmaxf(mk1, fabsf(__uint_as_float(wk & 0xFFFF0000u)));
        mv0 = fmaxf(mv0, fabsf(__uint_as_float(wv << 16)));
        mv1 = fmaxf(mv1, fabsf(__uint_as_float(wv & 0xFFFF0000u)));
      }
      // non-negative floats order like their bit patterns
      atomicMax(reinterpret_cast<unsigned int*>(kav), __float_as_uint(mk0));
      atomicMax(reinterpret_cast<unsigned int*>(kav + 1), __float_as_uint(mk1));
      atomicMax(reinterpret_cast<unsigned int*>(vav), __float_as_uint(mv0));
      atomicMax(reinterpret_cast<unsigned int*>(vav + 1), __float_as_uint(mv1));
    } else {
      const float sk0 = kav[0] / 127.f, sk1 = kav[1] / 127.f;
      const float sv0 = vav[0] / 127.f, sv1 = vav[1] / 127.f;
      const int64_t R_l = (layer_base[l + 1] - layer_base[l]) / (int64_t(p.B) * p.D);
      const int64_t dst_row0 = int64_t(b) * R_l + head_off[l * H + h] + seg_off[(l * H + h) * S + s] + r0;
      int8_t* kd = kq + layer_base[l] + dst_row0 * p.D + 2 * col;
      int8_t* vd = vq + layer_base[l] + dst_row0 * p.D + 2 * col;
      auto code = [](float x, float sc) -> int {
        if (sc == 0.f) return 0;
        const float t = rintf(__fdiv_rn(x, sc));
        return int(fminf(fmaxf(t, -127.f), 127.f));
      };
      for (int r = rofs; r < nrows; r += rstep) {
        const uint32_t wk = *reinterpret_cast<const uint32_t*>(ks + int64_t(r) * p.D);
        const uint32_t wv = *reinterpret_cast<const uint32_t*>(vs + int64_t(r) * p.D);
        const int k0 = code(__uint_as_float(wk << 16), sk0), k1 = code(__uint_as_float(wk & 0xFFFF0000u), sk1);
        const int v0 = code(__uint_as_float(wv << 16), sv0), v1 = code(__uint_as_float(wv & 0xFFFF0000u), sv1);
        *reinterpret_cast<uint16_t*>(kd + int64_t(r) * p.D) = uint16_t((k0 & 0xFF) | ((k1 & 0xFF) << 8));
        *reinterpret_cast<uint16_t*>(vd + int64_t(r) * p.D) = uint16_t((v0 & 0xFF) | ((v1 & 0xFF) << 8));
      }
    }
  }
}

// Dequantisation of one layer: one warp per row of the layer's compacted
// block, 4 channels per lane; the row's (b, h, scale) comes from the layer's
// offset tables, x' = code * (absmax / 127) rounded to bf16.
struct DequantParams {
  ScaleTable sc;
  int B, H, D;
  int64_t rows;            // B * R_l
};

__global__ void __launch_bounds__(256) dequant_kernel(const int8_t* __restrict__ kq, const int8_t* __restrict__ vq,
                                                      const float* __restrict__ ka, const float* __restrict__ va,
                                                      DequantParams p, const int32_t* __restrict__ head_off,
                                                      const int32_t* __restrict__ seg_off, uint16_t* __restrict__ kc,
                                                      uint16_t* __restrict__ vc) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x / 32);
  const int64_t R = p.rows / p.B;
  const int S = p.sc.S;
  for (int64_t row = int64_t(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); row < p.rows; row += warps) {
    const int b = int(row / R);
    const int64_t rr = row - int64_t(b) * R;
    int lo = 0, hi = p.H;                 // head: last h with head_off[h] <= rr
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (head_off[mid] <= rr) lo = mid; else hi = mid;
    }
    // heads that keep nothing share head_off with the next head: take the last
    while (lo + 1 < p.H && head_off[lo + 1] <= rr) ++lo;
    const int h = lo;
    const int64_t within = rr - head_off[h];
    int sc = -1;
    for (int s = 0; s < S; ++s) {
      const int32_t so = seg_off[h * S + s];
      if (so >= 0 && within >= so && within < so + p.sc.n[s]) sc = s;
    }
    if (sc < 0) continue;
    const int64_t arow = ((int64_t(b) * p.H + h) * S + sc) * p.D;
    for (int d = lane * 4; d < p.D; d += 128) {
      const uint32_t ck = *reinterpret_cast<const uint32_t*>(kq + row * p.D + d);
      const uint32_t cv = *reinterpret_cast<const uint32_t*>(vq + row * p.D + d);
      const float4 ak = *reinterpret_cast<const float4*>(ka + arow + d);
      const float4 av = *reinterpret_cast<const float4*>(va + arow + d);
      auto x = [](uint32_t w, int i) { return float(int8_t((w >> (8 * i)) & 0xFF)); };
      uint2 ok, ov;
      ok.x = pack_bf16x2(x(ck, 0) * (ak.x / 127.f), x(ck, 1) * (ak.y / 127.f));
      ok.y = pack_bf16x2(x(ck, 2) * (ak.z / 127.f), x(ck, 3) * (ak.w / 127.f));
      ov.x = pack_bf16x2(x(cv, 0) * (av.x / 127.f), x(cv, 1) * (av.y / 127.f));
      ov.y = pack_bf16x2(x(cv, 2) * (av.z / 127.f), x(cv, 3) * (av.w / 127.f));
      *reinterpret_cast<uint2*>(kc + row * p.D + d) = ok;
      *reinterpret_cast<uint2*>(vc + row * p.D + d) = ov;
    }
  }
}

}  // namespace vark

using namespace vark;

extern "C" int vark_quantize_kv_int8(const uint16_t* k, const uint16_t* v, int64_t layer_stride, int L, int B, int H,
                                     int S, int D, const int32_t* sides, const uint8_t* keep,
                                     const int32_t* head_off, const int32_t* seg_off, const int64_t* layer_base,
                                     int8_t* kq, int8_t* vq, float* k_absmax, float* v_absmax, void* stream) {
  if (!k || !v || !keep || !head_off || !seg_off || !layer_base || !kq || !vq || !k_absmax || !v_absmax)
    return VARK_E_ARG;
  QuantParams q;
  CompactParams& p = q.c;
  int rc = make_scale_table(S, sides, &p.sc);
  if (rc) return rc;
  if (L < 1 || H < 1 || B < 1 || D < 8 || D % 8 != 0 || D > 512) return VARK_E_SHAPE;
  if (H > kMaxGroupLH) return VARK_E_SHAPE;
  if (layer_stride < int64_t(B) * H * p.sc.T * D) return VARK_E_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(kq) || !aligned16(vq) || !aligned16(k_absmax) ||
      !aligned16(v_absmax))
    return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t nabs = int64_t(L) * B * H * S * D;
  if (cudaMemsetAsync(k_absmax, 0, size_t(nabs) * 4, st) != cudaSuccess ||
      cudaMemsetAsync(v_absmax, 0, size_t(nabs) * 4, st) != cudaSuccess)
    return VARK_E_CUDA;
  p.L = L; p.B = B; p.H = H; p.D = D; p.layer_stride = layer_stride; p.src_rows = p.sc.T;
  p.src_head_off = nullptr; p.src_seg_off = nullptr; p.src_layer_base = nullptr;
  for (int s = 0; s < VARK_MAX_SCALES; ++s) {
    p.chunks[s] = s < S ? (p.sc.n[s] + kChunkRows - 1) / kChunkRows : 0;
    p.src_off[s] = s < S ? p.sc.off[s] : 0;
  }
  q.scale_stride_l = int64_t(B) * H * S * D;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int layers_per_group = std::max(1, kMaxGroupLH / H);
  for (int mode = 0; mode < 2; ++mode) {
    q.mode = mode;
    for (int l0 = 0; l0 < L; l0 += layers_per_group) {
      p.l0 = l0;
      p.nl = std::min(layers_per_group, L - l0);
      quant_kernel<<<nsm * 4, kQuantThreads, 0, st>>>(k, v, q, keep, head_off, seg_off, layer_base, kq, vq,
                                                      k_absmax, v_absmax);
      if (cudaGetLastError() != cudaSuccess) return VARK_E_CUDA;
    }
  }
  return VARK_OK;
}

extern "C" int vark_dequantize_layer_int8(const int8_t* kq, const int8_t* vq, const float* k_absmax,
                                          const float* v_absmax, int64_t kc_rows, int B, int H, int S, int D,
                                          const int32_t* sides, const int32_t* head_off, const int32_t* seg_off,
                                          uint16_t* kc, uint16_t* vc, void* stream) {
  if (!kq || !vq || !k_absmax || !v_absmax || !head_off || !seg_off || !kc || !vc) return VARK_E_ARG;
  DequantParams p;
  int rc = make_scale_table(S, sides, &p.sc);
  if (rc) return rc;
  if (B < 1 || H < 1 || D < 4 || D % 4 != 0 || D > 512 || kc_rows < 0 || kc_rows % B != 0) return VARK_E_SHAPE;
  if (!aligned16(k_absmax) || !aligned16(v_absmax) || (reinterpret_cast<uintptr_t>(kq) & 3) ||
      (reinterpret_cast<uintptr_t>(vq) & 3) || !aligned16(kc) || !aligned16(vc))
    return VARK_E_ALIGN;
  if ((rc = check_device_sm100())) return rc;
  if (kc_rows == 0) return VARK_OK;
  p.B = B; p.H = H; p.D = D; p.rows = kc_rows;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  dequant_kernel<<<nsm * 8, 256, 0, static_cast<cudaStream_t>(stream)>>>(kq, vq, k_absmax, v_absmax, p, head_off,
                                                                          seg_off, kc, vc);
  return cudaGetLastError() == cudaSuccess ? VARK_OK : VARK_E_CUDA;
}
