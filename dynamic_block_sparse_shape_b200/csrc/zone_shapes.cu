// a1 + a2: macro-zone statistics and the per-zone block shape.
//
// Prism README, "Overview": each zone's local structure is estimated from the
// video features' variance along the channel and from the a2v cross-attention
// norms, and each zone gets a block shape that is finer along axes of fast
// visual change and strong audio-visual coupling. Prism walkthrough
// (wmrh.cn/news/72296), section "桥接残差反哺稀疏注意力": the per-token L2 norm of
// the unscaled a2v residual is the audio-influence proxy; sounding regions get
// finer blocks. The rule itself (documented in include/prism.h) is this
// library's reading; the pages print no formula.
//
// Kernels:
//   feat_stats   persistent; a TMA 4-D box brings one zone x 128-byte channel
//                slice into shared memory per stage; 8 warps each own one of
//                {t, h, w line sums, plain sum of squares} x {even, odd
//                lines}; lanes own one 4-byte word (2 bf16 / 1 fp32 channels).
//   feat_stats8  the same statistics for 8 x 8 x 8 zones: 16 compute warps
//                over t-slices and h-planes, 16-byte shared loads, fixed
//                strides (the general kernel serves every other zone shape).
//   res_norm     one warp per token: r(n) = ||res[n, :]||_2 in fp32.
//   zone_res     one CTA per zone: line variances of r along t/h/w (fp64) and
//                the zone sum of r.
//   choose       one warp per zone: grid mean of r (every CTA, same order),
//                the zone's chunk partials, then the costs in fp64, argmin
//                (ties to the lower index) and margin.
#include <cuda_bf16.h>

#include <algorithm>
#include <cfloat>
#include <cmath>
#include <mutex>

#include "host.h"
#include "ptx.cuh"

namespace prism {
namespace {

constexpr int kFeatStages = 3;
constexpr int kFeatThreads = 288;  // 8 compute warps + 1 TMA warp

template <int ES>
__device__ __forceinline__ float2 load_word(const uint8_t* p) {
  if constexpr (ES == 2) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
  } else {
    return make_float2(*reinterpret_cast<const float*>(p), 0.f);
  }
}

template <int ES>
__global__ void __launch_bounds__(kFeatThreads, 1)
    feat_stats_kernel(const __grid_constant__ CUtensorMap fmap, const Geo g, int n_chunks, float* __restrict__ partial,
                      int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full_bar[kFeatStages], empty_bar[kFeatStages];
  const int zvol = g.Zt * g.Zh * g.Zw;
  const uint32_t tile_bytes = uint32_t(zvol) * 128u;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = g.n_zones * n_chunks;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFeatStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 8);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 8) {
    if (lane == 0) {
      tma_prefetch_desc(&fmap);
      int k = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++k) {
        const int s = k % kFeatStages;
        if (!mbar_wait(&empty_bar[s], ((k / kFeatStages) & 1) ^ 1, status)) break;
        const int z = tile / n_chunks, c = tile - z * n_chunks;
        const int zt = z / (g.nzh * g.nzw), zr = z - zt * g.nzh * g.nzw;
        const int zh = zr / g.nzw, zw = zr - zh * g.nzw;
        mbar_arrive_expect_tx(&full_bar[s], tile_bytes);
        tma_load_4d(smem + size_t(s) * tile_bytes, &fmap, &full_bar[s], c * (128 / ES), zw * g.Zw, zh * g.Zh,
                    zt * g.Zt);
      }
    }
    return;
  }
  // compute warps: warp = kind * 2 + part
  const int kind = warp >> 1, part = warp & 1;
  const int HW = g.Zh * g.Zw;
  int k = 0;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++k) {
    const int s = k % kFeatStages;
    if (!mbar_wait(&full_bar[s], (k / kFeatStages) & 1, status)) break;
    const uint8_t* base = smem + size_t(s) * tile_bytes + lane * 4;
    float acc = 0.f;
    if (kind == 3) {
#pragma unroll 8
      for (int r = part; r < zvol; r += 2) {
        const float2 x = load_word<ES>(base + r * 128);
        acc = fmaf(x.x, x.x, fmaf(x.y, x.y, acc));
      }
    } else {
      const int La = kind == 0 ? g.Zt : (kind == 1 ? g.Zh : g.Zw);
      const int nlines = zvol / La;
      for (int line = part; line < nlines; line += 2) {
        int r0, step;
        if (kind == 0) {  // line = (h, w): rows line + i*HW
          r0 = line;
          step = HW;
        } else if (kind == 1) {  // line = (t, w): rows t*HW + i*Zw + w
          const int t = line / g.Zw, w = line - t * g.Zw;
          r0 = t * HW + w;
          step = g.Zw;
        } else {  // line = (t, h): rows line*Zw + i
          r0 = line * g.Zw;
          step = 1;
        }
        float s0 = 0.f, s1 = 0.f;
        for (int i0 = 0; i0 < La; i0 += 8) {
          float2 x[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)  // eight independent shared loads in flight
            x[i] = i0 + i < La ? load_word<ES>(base + (r0 + (i0 + i) * step) * 128) : make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            s0 += x[i].x;
            s1 += x[i].y;
          }
        }
        acc = fmaf(s0, s0, fmaf(s1, s1, acc));
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    __syncwarp();
    if (lane == 0) {
      partial[size_t(tile) * 8 + warp] = acc;
      mbar_arrive(&empty_bar[s]);
    }
  }
}

// The same statistics for 8 x 8 x 8 zones, with fixed strides and 16-byte
// shared loads. 16 compute warps: warp k < 8 owns the t-slice t = k (sum of
// squares, the line sums along w and along h of that slice), warp 8 + k the
// h-plane h = k (line sums along t). A lane owns one 16-byte channel group
// (cg = lane % 8) of rows w = q and w = q + 4 (q = lane / 8), so one load
// instruction covers four rows. The 16 warps' sums are combined in a fixed
// order by warp 0 (deterministic) into the per-tile layout {t, h, w, x^2}
// (slots 2 * kind; slots 2 * kind + 1 are zero).
constexpr int kFeat8Warps = 16;
constexpr int kFeat8Threads = 32 * (kFeat8Warps + 1);

template <int ES>
__device__ __forceinline__ void unpack16(const uint4 u, float* x) {
  if constexpr (ES == 2) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    x[0] = __uint_as_float(u.x);
    x[1] = __uint_as_float(u.y);
    x[2] = __uint_as_float(u.z);
    x[3] = __uint_as_float(u.w);
  }
}

template <int ES>
__global__ void __launch_bounds__(kFeat8Threads, 1)
    feat_stats8_kernel(const __grid_constant__ CUtensorMap fmap, const Geo g, int n_chunks, float* __restrict__ partial,
                       int* status) {
  constexpr int CPL = 16 / ES;        // channels per lane
  constexpr uint32_t kTile = 512 * 128;  // one zone x 128-byte channel slice
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* red = reinterpret_cast<float*>(smem + kFeatStages * kTile);  // [stage][warp][4]
  __shared__ uint64_t full_bar[kFeatStages], empty_bar[kFeatStages], red_bar[kFeatStages];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = g.n_zones * n_chunks;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFeatStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], kFeat8Warps);
      mbar_init(&red_bar[s], kFeat8Warps);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == kFeat8Warps) {
    if (lane == 0) {
      tma_prefetch_desc(&fmap);
      int k = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++k) {
        const int s = k % kFeatStages;
        if (!mbar_wait(&empty_bar[s], ((k / kFeatStages) & 1) ^ 1, status)) break;
        const int z = tile / n_chunks, c = tile - z * n_chunks;
        const int zt = z / (g.nzh * g.nzw), zr = z - zt * g.nzh * g.nzw;
        const int zh = zr / g.nzw, zw = zr - zh * g.nzw;
        mbar_arrive_expect_tx(&full_bar[s], kTile);
        tma_load_4d(smem + size_t(s) * kTile, &fmap, &full_bar[s], c * (128 / ES), zw * 8, zh * 8, zt * 8);
      }
    }
    return;
  }
  const int q = lane >> 3, cg = lane & 7;
  const bool slice = warp < 8;  // t-slice (true) or h-plane (false)
  const int k8 = warp & 7;
  int k = 0;
  for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++k) {
    const int s = k % kFeatStages;
    if (!mbar_wait(&full_bar[s], (k / kFeatStages) & 1, status)) break;
    const uint8_t* base = smem + size_t(s) * kTile + cg * 16;
    float col[2][CPL];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < CPL; ++c) col[a][c] = 0.f;
    float a_sq = 0.f, a_w = 0.f, a_col = 0.f;
    if (slice) {
      // rows t*64 + 4i + q: h = i / 2, w = 4 (i % 2) + q
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        float x0[CPL], x1[CPL], rp[CPL];
        unpack16<ES>(*reinterpret_cast<const uint4*>(base + (k8 * 64 + 8 * h + q) * 128), x0);
        unpack16<ES>(*reinterpret_cast<const uint4*>(base + (k8 * 64 + 8 * h + 4 + q) * 128), x1);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          a_sq = fmaf(x0[c], x0[c], fmaf(x1[c], x1[c], a_sq));
          col[0][c] += x0[c];
          col[1][c] += x1[c];
          rp[c] = x0[c] + x1[c];
        }
        // line sum along w of (t, h): the four q-lanes of this channel group
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          rp[c] += __shfl_xor_sync(0xffffffffu, rp[c], 8);
          rp[c] += __shfl_xor_sync(0xffffffffu, rp[c], 16);
        }
        if (q == 0) {
#pragma unroll
          for (int c = 0; c < CPL; ++c) a_w = fmaf(rp[c], rp[c], a_w);
        }
      }
    } else {
      // rows t*64 + h*8 + 4 (i % 2) + q with t = i / 2: the columns are the t-lines
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        float x0[CPL], x1[CPL];
        unpack16<ES>(*reinterpret_cast<const uint4*>(base + (t * 64 + k8 * 8 + q) * 128), x0);
        unpack16<ES>(*reinterpret_cast<const uint4*>(base + (t * 64 + k8 * 8 + 4 + q) * 128), x1);
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          col[0][c] += x0[c];
          col[1][c] += x1[c];
        }
      }
    }
    // column sums are complete line sums (along h for a t-slice, along t for an h-plane)
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int c = 0; c < CPL; ++c) a_col = fmaf(col[a][c], col[a][c], a_col);
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      a_sq += __shfl_xor_sync(0xffffffffu, a_sq, o);
      a_w += __shfl_xor_sync(0xffffffffu, a_w, o);
      a_col += __shfl_xor_sync(0xffffffffu, a_col, o);
    }
    float* rs = red + (s * kFeat8Warps + warp) * 4;
    if (lane == 0) {
      rs[0] = a_col;  // t-slice: h-lines; h-plane: t-lines
      rs[1] = a_w;
      rs[2] = a_sq;
      mbar_arrive(&red_bar[s]);
    }
    if (warp == 0) {
      // combine the 16 warps in a fixed order; the tile's stage is released after it
      if (lane == 0) {
        const bool ok = mbar_wait(&red_bar[s], (k / kFeatStages) & 1, status);
        const float* r = red + s * kFeat8Warps * 4;
        float st = 0.f, sh = 0.f, sw = 0.f, sq = 0.f;
        for (int w = 0; w < 8; ++w) {
          sh += r[w * 4 + 0];
          sw += r[w * 4 + 1];
          sq += r[w * 4 + 2];
          st += r[(8 + w) * 4 + 0];
        }
        float* p = partial + size_t(tile) * 8;
        p[0] = ok ? st : 0.f;
        p[1] = 0.f;
        p[2] = ok ? sh : 0.f;
        p[3] = 0.f;
        p[4] = ok ? sw : 0.f;
        p[5] = 0.f;
        p[6] = ok ? sq : 0.f;
        p[7] = 0.f;
      }
      __syncwarp();
    }
    if (lane == 0) mbar_arrive(&empty_bar[s]);
  }
}

template <int ES>
__global__ void __launch_bounds__(256) res_norm_kernel(const uint8_t* __restrict__ res, int64_t ld_bytes, int row_bytes,
                                                       int n_tokens, float* __restrict__ r) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= n_tokens) return;
  const uint8_t* row = res + int64_t(warp) * ld_bytes;
  float acc = 0.f;
  const int n16 = row_bytes / 16;
#pragma unroll 4
  for (int j = lane; j < n16; j += 32) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row) + j);
    if constexpr (ES == 2) {
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xFFFF0000u);
        acc = fmaf(lo, lo, fmaf(hi, hi, acc));
      }
    } else {
      const float f[4] = {__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w)};
#pragma unroll
      for (int q = 0; q < 4; ++q) acc = fmaf(f[q], f[q], acc);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) r[warp] = sqrtf(acc);
}

// One CTA (256 threads) per zone: A_a = mean over lines || a of the
// population variance of r along the line (fp64), and the zone sum of r.
__global__ void __launch_bounds__(256) zone_res_kernel(const Geo g, const float* __restrict__ r,
                                                       double* __restrict__ zres) {
  __shared__ float rz[kMaxZoneTokens];
  __shared__ double red[4][8];
  const int z = blockIdx.x;
  const int zt = z / (g.nzh * g.nzw), zr = z - zt * g.nzh * g.nzw;
  const int zh = zr / g.nzw, zw = zr - zh * g.nzw;
  // the zone's extents clipped to the grid (whole zones: Zt, Zh, Zw)
  int Et, Eh, Ew;
  zone_extents(g, z, &Et, &Eh, &Ew);
  const int zvol = Et * Eh * Ew, HW = Eh * Ew;
  for (int i = threadIdx.x; i < zvol; i += blockDim.x) {
    const int t = i / HW, h = (i / Ew) % Eh, w = i % Ew;
    rz[i] = r[((zt * g.Zt + t) * g.H + zh * g.Zh + h) * g.W + zw * g.Zw + w];
  }
  __syncthreads();
  double acc[4] = {0, 0, 0, 0};
  for (int a = 0; a < 3; ++a) {
    const int La = a == 0 ? Et : (a == 1 ? Eh : Ew);
    const int nlines = zvol / La;
    for (int line = threadIdx.x; line < nlines; line += blockDim.x) {
      int r0, step;
      if (a == 0) { r0 = line; step = HW; }
      else if (a == 1) { const int t = line / Ew; r0 = t * HW + (line - t * Ew); step = Ew; }
      else { r0 = line * Ew; step = 1; }
      double mean = 0;
      for (int i = 0; i < La; ++i) mean += rz[r0 + i * step];
      mean /= La;
      double var = 0;
      for (int i = 0; i < La; ++i) {
        const double d = rz[r0 + i * step] - mean;
        var += d * d;
      }
      acc[a] += var / La / nlines;
    }
  }
  for (int i = threadIdx.x; i < zvol; i += blockDim.x) acc[3] += rz[i];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int q = 0; q < 4; ++q) {
    double v = acc[q];
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[q][warp] = v;
  }
  __syncthreads();
  if (threadIdx.x < 4) {
    double v = 0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) v += red[threadIdx.x][w];
    zres[size_t(z) * 4 + threadIdx.x] = v;
  }
}

// One warp per zone (8 zones per CTA). Every CTA first forms the grid mean of
// r from the per-zone sums in the same fixed order (so all CTAs agree), then
// each warp sums its zone's per-chunk partials (lanes over chunks, fp64) and
// lane 0 evaluates the costs.
constexpr int kChooseWarps = 8;
__global__ void __launch_bounds__(32 * kChooseWarps) choose_kernel(const Geo g, const float* __restrict__ partial,
                                                                   int n_chunks, int feat_c,
                                                                   const double* __restrict__ zres, int have_feat,
                                                                   int have_res, float w_audio, float gamma,
                                                                   float gate_max, int32_t* __restrict__ zone_shape,
                                                                   float* __restrict__ zone_margin,
                                                                   const int* __restrict__ status) {
  __shared__ double red[32 * kChooseWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  double s = 0;
  if (have_res)
    for (int z = tid; z < g.n_zones; z += blockDim.x) s += zres[size_t(z) * 4 + 3];
  red[tid] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w; w >>= 1) {
    if (tid < w) red[tid] += red[tid + w];
    __syncthreads();
  }
  const double mbar = red[0] / (double(g.T) * g.H * g.W);
  const int z = blockIdx.x * kChooseWarps + warp;
  if (z >= g.n_zones) return;
  double q[4] = {0, 0, 0, 0};
  if (have_feat) {
    for (int c = lane; c < n_chunks; c += 32) {
      const float4 a = *reinterpret_cast<const float4*>(partial + (size_t(z) * n_chunks + c) * 8);
      const float4 b = *reinterpret_cast<const float4*>(partial + (size_t(z) * n_chunks + c) * 8 + 4);
      q[0] += double(a.x) + double(a.y);
      q[1] += double(a.z) + double(a.w);
      q[2] += double(b.x) + double(b.y);
      q[3] += double(b.z) + double(b.w);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int o = 16; o; o >>= 1) q[k] += __shfl_xor_sync(0xffffffffu, q[k], o);
  }
  if (lane != 0) return;
  if (*reinterpret_cast<const volatile int*>(status) & kDevErrTimeout) {
    // a statistics kernel gave up waiting for its copies: its sums are incomplete
    zone_shape[z] = -1;
    if (zone_margin) zone_margin[z] = __int_as_float(0x7fc00000);
    return;
  }
  if (!have_feat && !have_res) {
    zone_shape[z] = 0;
    if (zone_margin) zone_margin[z] = INFINITY;
    return;
  }
  // line lengths and member count of the zone clipped to the grid; the channel
  // partial sums count only member tokens (the TMA copy fills the rest with 0)
  int Et, Eh, Ew;
  zone_extents(g, z, &Et, &Eh, &Ew);
  const double zvol = double(Et) * Eh * Ew;
  const double Z[3] = {double(Et), double(Eh), double(Ew)};
  double V[3] = {0, 0, 0}, A[3] = {0, 0, 0};
  if (have_feat)
    for (int a = 0; a < 3; ++a) V[a] = (q[3] - q[a] / Z[a]) / (zvol * feat_c);
  double gz = 0;
  if (have_res && mbar > 0) {
    for (int a = 0; a < 3; ++a) A[a] = zres[size_t(z) * 4 + a];
    const double m = zres[size_t(z) * 4 + 3] / zvol;
    gz = fmin(fmax(m / mbar - 1.0, 0.0), double(gate_max));
  }
  const double sv = V[0] + V[1] + V[2] + 1e-12, sa = A[0] + A[1] + A[2] + 1e-12;
  double S[3];
  for (int a = 0; a < 3; ++a) S[a] = 3.0 * V[a] / sv + double(w_audio) * gz * 3.0 * A[a] / sa;
  const double tot = S[0] + S[1] + S[2];
  for (int a = 0; a < 3; ++a) S[a] = tot > 0 ? 3.0 * S[a] / tot : 1.0;
  double best = INFINITY, second = INFINITY;
  int bi = 0;
  for (int c = 0; c < g.n_cand; ++c) {
    double cost = 0;
    for (int a = 0; a < 3; ++a) {
      const double e = log2(double(g.cand[c][a]));
      cost += S[a] * e + double(gamma) * (e - 2.0) * (e - 2.0);
    }
    if (cost < best) {
      second = best;
      best = cost;
      bi = c;
    } else if (cost < second) {
      second = cost;
    }
  }
  zone_shape[z] = bi;
  if (zone_margin) zone_margin[z] = float(second - best);
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// Channel line statistics of the features into `partial` ([tile][8], tile =
// zone * n_chunks + 128-byte channel slice): the fixed-stride kernel for
// 8 x 8 x 8 zones, the general one otherwise.
prism_status launch_feat_stats(const Geo& g, const void* feat, int64_t feat_ld, int feat_c, int fes, int n_chunks,
                               float* partial, int* status, cudaStream_t s) {
  CUtensorMap fmap;
  const uint64_t dims[4] = {uint64_t(feat_c), uint64_t(g.W), uint64_t(g.H), uint64_t(g.T)};
  const uint64_t strides[3] = {uint64_t(feat_ld) * fes, uint64_t(feat_ld) * fes * g.W,
                               uint64_t(feat_ld) * fes * g.W * g.H};
  const uint32_t box[4] = {uint32_t(128 / fes), uint32_t(g.Zw), uint32_t(g.Zh), uint32_t(g.Zt)};
  prism_status st = encode_tiled(&fmap, fes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                                 4, feat, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != PRISM_OK) return st;
  const int n_tiles = g.n_zones * n_chunks;
  const int grid = std::min(n_tiles, sm_count());
  if (g.Zt == 8 && g.Zh == 8 && g.Zw == 8) {
    const size_t smem = size_t(kFeatStages) * 512 * 128 + size_t(kFeatStages) * kFeat8Warps * 4 * sizeof(float) + 1024;
    if (fes == 2) {
      cudaFuncSetAttribute(feat_stats8_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      feat_stats8_kernel<2><<<grid, kFeat8Threads, smem, s>>>(fmap, g, n_chunks, partial, status);
    } else {
      cudaFuncSetAttribute(feat_stats8_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      feat_stats8_kernel<4><<<grid, kFeat8Threads, smem, s>>>(fmap, g, n_chunks, partial, status);
    }
  } else {
    const size_t smem = size_t(kFeatStages) * g.Zt * g.Zh * g.Zw * 128 + 1024;
    if (fes == 2) {
      cudaFuncSetAttribute(feat_stats_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      feat_stats_kernel<2><<<grid, kFeatThreads, smem, s>>>(fmap, g, n_chunks, partial, status);
    } else {
      cudaFuncSetAttribute(feat_stats_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      feat_stats_kernel<4><<<grid, kFeatThreads, smem, s>>>(fmap, g, n_chunks, partial, status);
    }
  }
  return cudaGetLastError() == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA;
}


struct ZoneWs {
  size_t partial, r, zres, total;
};

ZoneWs zone_ws_layout(const Geo& g, int feat_c, int feat_es, int res_c) {
  WsCarver c;
  ZoneWs w;
  const int n_chunks = feat_c > 0 ? feat_c * feat_es / 128 : 0;
  w.partial = c.take(size_t(g.n_zones) * std::max(n_chunks, 1) * 8 * sizeof(float));
  w.r = c.take(size_t(g.T) * g.H * g.W * sizeof(float) * (res_c > 0 ? 1 : 0) + 16);
  w.zres = c.take(size_t(g.n_zones) * 4 * sizeof(double));
  w.total = c.off;
  return w;
}

}  // namespace

size_t zone_shapes_ws_bytes(const Geo& g, int feat_c, prism_dtype feat_dtype, int res_c) {
  return zone_ws_layout(g, feat_c, feat_dtype == PRISM_FP32 ? 4 : 2, res_c).total;
}

int device_sm_count() { return sm_count(); }

}  // namespace prism

using namespace prism;

// ---------------------------------------------------------------------------
// Allocation-free variant of prism_zone_shapes. The scratch (per-zone channel
// partial sums, per-token residual norms, per-zone residual statistics and the
// status word) lives in one file-scope device array instead of a caller
// workspace. Host code only ever sees the array's host-side shadow, so the
// device address is looked up with cudaGetSymbolAddress, once per device and
// context: a new primary context (after cudaDeviceReset) reloads the module,
// which may place the array elsewhere, so the address is looked up again.
namespace prism {
namespace {

constexpr size_t kZoneStaticBytes = size_t(4) << 20;  // 4 MiB, held by every GPU that loads the library
static __device__ __align__(256) uint8_t g_zone_scratch[kZoneStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn g_ctx_get = nullptr;
std::once_flag g_ctx_once;

void load_ctx_get() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &fn, 12000, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_get = reinterpret_cast<CtxGetCurrentFn>(fn);
}

// Device address of g_zone_scratch in the current device's current context.
prism_status static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PRISM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PRISM_ERR_UNSUPPORTED;
  std::call_once(g_ctx_once, load_ctx_get);
  CUcontext ctx = nullptr;
  if (g_ctx_get && g_ctx_get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev] || !ctx || g_scratch_ctx[dev] != ctx) {
    // (no context known yet, or a new one: the lookup itself makes the primary context current)
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_zone_scratch) != cudaSuccess || !p) return PRISM_ERR_CUDA;
    if (g_ctx_get && g_ctx_get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  *out = g_scratch_ptr[dev];
  return PRISM_OK;
}

}  // namespace
}  // namespace prism

namespace {

// Where the scratch of a zone-shape call lives: the caller's workspace, or the
// library's static device array (prism_zone_shapes_static).
enum class ZoneScratch { kWorkspace, kStatic };

// Validation and the launch sequence shared by prism_zone_shapes and
// prism_zone_shapes_static; they differ only in where the scratch lives.
prism_status zone_shapes_run(const prism_geometry* geo, const void* feat, int64_t feat_ld, int32_t feat_c,
                             prism_dtype feat_dtype, const void* res, int64_t res_ld, int32_t res_c,
                             prism_dtype res_dtype, const prism_shape_params* params, int32_t* zone_shape,
                             float* zone_margin, ZoneScratch where, void* ws, size_t ws_bytes, void* stream) {
  Geo g;
  prism_status st = make_geo(geo, &g);
  if (st != PRISM_OK) return st;
  if (!zone_shape) return PRISM_ERR_ARG;
  const prism_shape_params def = {1.0f, 0.25f, 4.0f};
  const prism_shape_params p = params ? *params : def;
  if (!(p.gamma >= 0.f) || !(p.w_audio >= 0.f) || !(p.gate_max >= 0.f)) return PRISM_ERR_ARG;
  if (feat) {
    if (feat_dtype != PRISM_BF16 && feat_dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
    if (feat_c <= 0 || feat_c % 64 || feat_ld < feat_c || feat_ld % 8) return PRISM_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(feat) % 16) return PRISM_ERR_ARG;
  } else {
    feat_c = 0;
  }
  const int res_es = res_dtype == PRISM_FP32 ? 4 : 2;
  if (res) {
    if (res_dtype != PRISM_BF16 && res_dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
    if (res_c <= 0 || res_c % 8 || res_ld < res_c || res_ld % 8) return PRISM_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(res) % 16) return PRISM_ERR_ARG;
    if ((int64_t(res_c) * res_es) % 16) return PRISM_ERR_ARG;
  } else {
    res_c = 0;
  }
  const int fes = feat_dtype == PRISM_FP32 ? 4 : 2;
  const ZoneWs L = zone_ws_layout(g, feat_c, fes, res_c);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (where == ZoneScratch::kWorkspace) {
    if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < L.total) return PRISM_ERR_WORKSPACE;
  } else {
    if (L.total > kZoneStaticBytes) return PRISM_ERR_UNSUPPORTED;  // grid too large for the static scratch
    if ((st = static_scratch(&ws)) != PRISM_OK) return st;
    // the status word is the only scratch a kernel reads before writing it
    if (cudaMemsetAsync(ws_status(ws), 0, sizeof(int), s) != cudaSuccess) return PRISM_ERR_CUDA;
  }
  uint8_t* w8 = reinterpret_cast<uint8_t*>(ws);
  float* partial = reinterpret_cast<float*>(w8 + L.partial);
  float* r = reinterpret_cast<float*>(w8 + L.r);
  double* zres = reinterpret_cast<double*>(w8 + L.zres);
  int* status = ws_status(ws);
  const int N = g.T * g.H * g.W;
  const int n_chunks = feat_c * fes / 128;
  if (feat) {
    if ((st = launch_feat_stats(g, feat, feat_ld, feat_c, fes, n_chunks, partial, status, s)) != PRISM_OK) return st;
  }
  if (res) {
    const int blocks = (N + 7) / 8;
    if (res_es == 2)
      res_norm_kernel<2><<<blocks, 256, 0, s>>>(reinterpret_cast<const uint8_t*>(res), res_ld * res_es,
                                                res_c * res_es, N, r);
    else
      res_norm_kernel<4><<<blocks, 256, 0, s>>>(reinterpret_cast<const uint8_t*>(res), res_ld * res_es,
                                                res_c * res_es, N, r);
    zone_res_kernel<<<g.n_zones, 256, 0, s>>>(g, r, zres);
    if (cudaGetLastError() != cudaSuccess) return PRISM_ERR_CUDA;
  }
  choose_kernel<<<(g.n_zones + kChooseWarps - 1) / kChooseWarps, 32 * kChooseWarps, 0, s>>>(
      g, partial, n_chunks, feat_c, zres, feat != nullptr, res != nullptr, p.w_audio, p.gamma, p.gate_max,
      zone_shape, zone_margin, status);
  return cuda_status(cudaGetLastError());
}

}  // namespace

extern "C" prism_status prism_zone_shapes(const prism_geometry* geo, const void* feat, int64_t feat_ld, int32_t feat_c,
                                          prism_dtype feat_dtype, const void* res, int64_t res_ld, int32_t res_c,
                                          prism_dtype res_dtype, const prism_shape_params* params,
                                          int32_t* zone_shape, float* zone_margin, void* ws, size_t ws_bytes,
                                          void* stream) {
  return zone_shapes_run(geo, feat, feat_ld, feat_c, feat_dtype, res, res_ld, res_c, res_dtype, params, zone_shape,
                         zone_margin, ZoneScratch::kWorkspace, ws, ws_bytes, stream);
}

extern "C" prism_status prism_zone_shapes_static(const prism_geometry* geo, const void* feat, int64_t feat_ld,
                                                 int32_t feat_c, prism_dtype feat_dtype, const void* res,
                                                 int64_t res_ld, int32_t res_c, prism_dtype res_dtype,
                                                 const prism_shape_params* params, int32_t* zone_shape,
                                                 float* zone_margin, void* stream) {
  return zone_shapes_run(geo, feat, feat_ld, feat_c, feat_dtype, res, res_ld, res_c, res_dtype, params, zone_shape,
                         zone_margin, ZoneScratch::kStatic, nullptr, 0, stream);
}
