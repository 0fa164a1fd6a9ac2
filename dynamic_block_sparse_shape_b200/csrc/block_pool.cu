// a3: block partition and mean pooling ("block-level features", Prism README
// "Overview"; mean pooling as the block feature).
//
// One CTA per (block, tensor): each thread owns 8 consecutive channels of the
// token row [heads * head_dim] and walks the block's 64 tokens eight at a time
// (eight independent 16-byte loads in flight), accumulating in fp32. A block
// clipped by the grid's edge averages its member tokens; an empty one is NaN.
// The output layout is [heads, n_blocks, head_dim] fp32.
#include <cuda_bf16.h>

#include "host.h"

namespace prism {
namespace {

template <typename T>
__device__ __forceinline__ void load8(const T* p, float* x);

template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float* x) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float* x) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// Sum of the block's member rows over this thread's 8 channels. GUARD is false
// for a block wholly inside the grid: eight unconditional loads in flight.
template <typename T, bool GUARD>
__device__ __forceinline__ void sum_block_rows(const Geo& g, const BlockBox& bb, const T* base, int64_t tok_stride,
                                               uint64_t members, float* acc) {
  // Block extents divide 64, so they are powers of two: token r of the block
  // (raster t, h, w) is found with shifts.
  const int lw = __ffs(bb.bw) - 1, lhw = lw + __ffs(bb.bh) - 1;
  for (int r0 = 0; r0 < kBlockTokens; r0 += 8) {
    float x[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = r0 + i;
      const int rt = r >> lhw, rh = (r >> lw) & (bb.bh - 1), rw = r & (bb.bw - 1);
      const int64_t n = (int64_t(bb.t0 + rt) * g.H + bb.h0 + rh) * g.W + bb.w0 + rw;
      if (!GUARD || ((members >> r) & 1)) {
        load8<T>(base + n * tok_stride, x[i]);
      } else {
#pragma unroll
        for (int c = 0; c < 8; ++c) x[i][c] = 0.f;
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += x[i][c];
  }
}

template <typename T>
__global__ void __launch_bounds__(1024) pool_kernel(const Geo g, const int32_t* __restrict__ zone_shape,
                                                    const T* __restrict__ q, const T* __restrict__ k,
                                                    int64_t tok_stride, int head_dim, float* __restrict__ qp,
                                                    float* __restrict__ kp, int* status) {
  const int b = blockIdx.x;
  const T* src = blockIdx.y ? k : q;
  float* dst = blockIdx.y ? kp : qp;
  const int c0 = threadIdx.x * 8;
  const int head = c0 / head_dim, dd = c0 - head * head_dim;
  float* out = dst + (size_t(head) * g.n_blocks + b) * head_dim + dd;
  const int shape = zone_shape[zone_of_block(g, b)];
  if (shape < 0 || shape >= g.n_cand) {
    if (threadIdx.x == 0) atomicOr(status, kDevErrBounds);
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = __int_as_float(0x7fc00000);
    return;
  }
  const BlockBox bb = block_box(g, shape, b);
  // members: the box's slots inside the grid (all 64 unless the zone is clipped)
  const uint64_t members = g.partial ? block_slot_mask(g, bb) : ~uint64_t(0);
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  const T* base = src + c0;
  if (members == ~uint64_t(0))
    sum_block_rows<T, false>(g, bb, base, tok_stride, members, acc);
  else
    sum_block_rows<T, true>(g, bb, base, tok_stride, members, acc);
  // an empty block has no feature: NaN, which the selection reads as "absent"
  const int cnt = __popcll(members);
  const float inv = cnt ? 1.0f / float(cnt) : __int_as_float(0x7fc00000);
  reinterpret_cast<float4*>(out)[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  reinterpret_cast<float4*>(out)[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
}

}  // namespace
}  // namespace prism

using namespace prism;

extern "C" prism_status prism_block_pool(const prism_geometry* geo, const int32_t* zone_shape, const void* q,
                                         const void* k, prism_dtype dtype, int32_t heads, int32_t head_dim,
                                         int64_t tok_stride, float* q_pool, float* k_pool, void* ws,
                                         size_t ws_bytes, void* stream) {
  Geo g;
  prism_status st = make_geo(geo, &g);
  if (st != PRISM_OK) return st;
  if (!zone_shape || !q || !k || !q_pool || !k_pool) return PRISM_ERR_ARG;
  if (dtype != PRISM_BF16 && dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
  if (head_dim != 64 && head_dim != 128) return PRISM_ERR_UNSUPPORTED;
  if (heads < 1 || int64_t(heads) * head_dim > 8192) return PRISM_ERR_UNSUPPORTED;
  if (tok_stride < int64_t(heads) * head_dim || tok_stride % 8) return PRISM_ERR_ARG;
  const size_t es = dtype == PRISM_FP32 ? 4 : 2;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k) % 16) return PRISM_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(q_pool) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16) return PRISM_ERR_ARG;
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < kWsHeader) return PRISM_ERR_WORKSPACE;
  (void)es;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const dim3 grid(g.n_blocks, 2);
  const int threads = heads * head_dim / 8;
  if (dtype == PRISM_BF16)
    pool_kernel<__nv_bfloat16><<<grid, threads, 0, s>>>(g, zone_shape, static_cast<const __nv_bfloat16*>(q),
                                                         static_cast<const __nv_bfloat16*>(k), tok_stride, head_dim,
                                                         q_pool, k_pool, ws_status(ws));
  else
    pool_kernel<float><<<grid, threads, 0, s>>>(g, zone_shape, static_cast<const float*>(q),
                                                static_cast<const float*>(k), tok_stride, head_dim, q_pool, k_pool,
                                                ws_status(ws));
  return cuda_status(cudaGetLastError());
}
