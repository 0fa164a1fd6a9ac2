// Audio-norm bias of the key blocks, an optional input of the block scoring.
//
// Prism walkthrough (wmrh.cn/news/72296), section "桥接残差反哺稀疏注意力": the
// per-token L2 norm of the unscaled a2v bridge residual is the proxy of how
// strongly audio drives a visual region, it is read when BSA scores blocks,
// and sounding regions keep more attention. The library's reading:
//   b_J = beta * mean_{n in J} r(n) / mean_{all n} r(n),  r(n) = ||res[n, :]||_2.
//
// block_norm_kernel: one CTA per block, one warp per 8 of its 64 slots. A
//   token's sum of squares is a strided lane sum of 16-byte loads (fp32),
//   reduced by a fixed butterfly; the block sum adds the member tokens' norms
//   in a fixed order (a block clipped by the grid's edge has fewer than 64
//   members). Every residual row is read once: the kernel is an HBM stream.
// bias_normalize_kernel: one CTA. The grid mean of r is the sum of the block
//   sums over the token count, summed in fp64 in a fixed order; then
//   b_J = beta * (sum_J / members_J) / grid mean in place (0 for a zero
//   residual and for an empty block, which the selection never keeps).
#include <cuda_bf16.h>

#include <cmath>

#include "host.h"

namespace prism {
namespace {

constexpr int kNormWarps = 8;
constexpr int kNormTokensPerWarp = kBlockTokens / kNormWarps;
constexpr int kNormalizeThreads = 1024;

template <int ES>
__device__ __forceinline__ float row_sum_squares(const uint8_t* row, int n16, int lane) {
  float acc = 0.f;
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
  return acc;
}

template <int ES>
__global__ void __launch_bounds__(kNormWarps * 32) block_norm_kernel(const Geo g, const int32_t* __restrict__ zone_shape,
                                                                     const uint8_t* __restrict__ res, int64_t ld_bytes,
                                                                     int row_bytes, float* __restrict__ out,
                                                                     int* status) {
  __shared__ float part[kNormWarps];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int shape = zone_shape[zone_of_block(g, b)];
  if (shape < 0 || shape >= g.n_cand) {
    if (threadIdx.x == 0) {
      atomicOr(status, kDevErrBounds);
      out[b] = __int_as_float(0x7fc00000);
    }
    return;
  }
  const BlockBox bb = block_box(g, shape, b);
  // Block extents divide 64, so they are powers of two: token r of the block
  // (raster t, h, w) is found with shifts.
  const int lw = __ffs(bb.bw) - 1, lhw = lw + __ffs(bb.bh) - 1;
  const int n16 = row_bytes / 16;
  const uint64_t members = g.partial ? block_slot_mask(g, bb) : ~uint64_t(0);
  float sum = 0.f;
  for (int i = 0; i < kNormTokensPerWarp; ++i) {
    const int r = warp * kNormTokensPerWarp + i;
    if (!((members >> r) & 1)) continue;  // warp-uniform
    const int rt = r >> lhw, rh = (r >> lw) & (bb.bh - 1), rw = r & (bb.bw - 1);
    const int64_t n = (int64_t(bb.t0 + rt) * g.H + bb.h0 + rh) * g.W + bb.w0 + rw;
    sum += sqrtf(row_sum_squares<ES>(res + n * ld_bytes, n16, lane));
  }
  if (lane == 0) part[warp] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kNormWarps; ++w) t += part[w];
    out[b] = t;  // the block's sum of r over its members
  }
}

__global__ void __launch_bounds__(kNormalizeThreads) bias_normalize_kernel(const Geo g,
                                                                           const int32_t* __restrict__ zone_shape,
                                                                           float* __restrict__ bias, float beta) {
  __shared__ double red[kNormalizeThreads];
  const int tid = threadIdx.x, nb = g.n_blocks;
  double s = 0.0;
  for (int j = tid; j < nb; j += kNormalizeThreads) s += double(bias[j]);
  red[tid] = s;
  __syncthreads();
  for (int half = kNormalizeThreads / 2; half; half >>= 1) {
    if (tid < half) red[tid] += red[tid + half];
    __syncthreads();
  }
  const double mean = red[0] / (double(g.T) * g.H * g.W);
  for (int j = tid; j < nb; j += kNormalizeThreads) {
    int members = kBlockTokens;
    if (g.partial) {
      const int sh = zone_shape[zone_of_block(g, j)];
      members = (sh >= 0 && sh < g.n_cand) ? __popcll(block_slot_mask(g, block_box(g, sh, j))) : 0;
    }
    float v;
    if (!(mean >= 0.0)) v = __int_as_float(0x7fc00000);  // NaN: a block reported an error
    else if (mean == 0.0 || members == 0) v = 0.f;
    else v = float(double(beta) * (double(bias[j]) / members) / mean);
    bias[j] = v;
  }
}

}  // namespace
}  // namespace prism

using namespace prism;

extern "C" prism_status prism_block_audio_bias(const prism_geometry* geo, const int32_t* zone_shape, const void* res,
                                               int64_t res_ld, int32_t res_c, prism_dtype res_dtype, float beta,
                                               float* key_bias, void* ws, size_t ws_bytes, void* stream) {
  Geo g;
  prism_status st = make_geo(geo, &g);
  if (st != PRISM_OK) return st;
  if (!zone_shape || !res || !key_bias) return PRISM_ERR_ARG;
  if (res_dtype != PRISM_BF16 && res_dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
  if (res_c <= 0 || res_c % 8 || res_ld < res_c || res_ld % 8) return PRISM_ERR_ARG;
  if (!std::isfinite(beta)) return PRISM_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(res) % 16 || reinterpret_cast<uintptr_t>(key_bias) % 4) return PRISM_ERR_ARG;
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < kWsHeader) return PRISM_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int es = res_dtype == PRISM_FP32 ? 4 : 2;
  const int64_t ld_bytes = res_ld * es;
  const int row_bytes = res_c * es;
  const uint8_t* r = static_cast<const uint8_t*>(res);
  if (es == 2)
    block_norm_kernel<2><<<g.n_blocks, kNormWarps * 32, 0, s>>>(g, zone_shape, r, ld_bytes, row_bytes, key_bias,
                                                                ws_status(ws));
  else
    block_norm_kernel<4><<<g.n_blocks, kNormWarps * 32, 0, s>>>(g, zone_shape, r, ld_bytes, row_bytes, key_bias,
                                                                ws_status(ws));
  bias_normalize_kernel<<<1, kNormalizeThreads, 0, s>>>(g, zone_shape, key_bias, beta);
  return cuda_status(cudaGetLastError());
}
