// a4 + a5: block scoring and hybrid top-k + cumulative-mass selection.
//
// Prism walkthrough (wmrh.cn/news/72296), section "三者如何协同": the gating
// step keeps the k highest-scoring blocks, then extends along the CDF of the
// block scores until cdf_threshold (default 0.20). Prism README "Overview":
// the hybrid rule sets each query's sparsity. Sol-Attn abstract on the Prism
// paper page: computing and materialising the proxy scores is the routing
// overhead, so the scores here live only in shared memory.
//
// select_kernel: one CTA = 8 query blocks of one head; 4 when more than 6912
// key blocks' logits must fit in shared memory. Two warps per row compute the
// logits, then select: each takes one half of the row, and the row's sums,
// counts and maxima combine through shared memory at a 64-thread barrier.
//   1. logits s_J = scale * qbar_I . kbar_J (+ b_J, the optional key-block
//      bias, walkthrough section "桥接残差反哺稀疏注意力") for all J, fp32 FFMA:
//      a thread streams four keys of the workspace's transposed pooled keys
//      (coalesced 512-byte warp reads per channel) and forms their logits
//      against the CTA's rows (shared-memory broadcasts);
//   2. per row: max, p_J = exp(s_J - max) in place as a ranking key (float
//      bits + 1; 0 for a NaN logit, which marks an absent block: an empty
//      block of a grid clipped at its edge), Z = sum p (fp64);
//   3. the mass threshold: bisection on the keys for
//      u* = max{u : sum_{key_J >= u} p_J >= tau * Z}; ties at u* are taken in
//      ascending J until the mass is reached -> m*;
//   4. m = max(k, m*); if m > m*, a bisection on counts finds the m-th key;
//      k and tau are the row's head's (per-head settings, walkthrough section
//      "实际案例与上手参考": the top-k part of the selection is a tunable ratio);
//   5. the kept set (ranked by p descending, ties to the lower J) is written
//      as a bitmask row with warp ballots, and kept[row] = m.
// transpose_keys_kernel: k_pool per head into key-major order in the workspace.
// scan_kernel: exclusive scan of kept into the CSR row_ptr (one CTA).
// fill_kernel: one warp per row expands the bitmask into ascending col_idx.
#include <algorithm>
#include <cfloat>
#include <cmath>

#include "host.h"
#include "ptx.cuh"

namespace prism {
namespace {

// Rows of logits per CTA live in shared memory: 8 rows up to 6912 key blocks,
// 4 rows (half the threads) up to 10240 (the 2K latent grid has 7680).
constexpr int kSelMaxBlocks8 = 6912;
constexpr int kSelMaxBlocks = 10240;
constexpr int kSelMaxHeads = 128;  // per-head settings passed as a kernel parameter

// Per-head floor k and mass threshold tau (uniform when per_head == 0).
struct SelHeads {
  int per_head;
  int k0;
  float tau0;
  int k[kSelMaxHeads];
  float tau[kSelMaxHeads];
};

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_i(int v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Row entries are kept as ranking keys: key = (float bits of p) + 1 for a
// present key block and 0 for an absent one (NaN logit: an empty block, or a
// NaN input). For p >= 0 the float bits order like the values, so keys order
// like p with every absent block below every present one.
__device__ __forceinline__ float key_value(uint32_t key) { return __uint_as_float(key - 1u); }

// Mass of the entries whose key is >= u >= 1: four independent fp32 chains per
// lane (at most nb/128 terms each, relative error below 2e-6 of the row's
// mass for 10240 entries), combined in fp64 and warp-reduced in a fixed order.
// The row total Z is this function at u = 1, so the bisection's invariant
// mass(>= 1) = Z >= tau Z holds exactly.
__device__ __forceinline__ double mass_at_least(const uint32_t* p, int jb, int nb, uint32_t u, int lane) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  int j = jb + lane;
  for (; j + 96 < nb; j += 128) {
    const uint32_t k0 = p[j], k1 = p[j + 32], k2 = p[j + 64], k3 = p[j + 96];
    a0 += k0 >= u ? key_value(k0) : 0.f;
    a1 += k1 >= u ? key_value(k1) : 0.f;
    a2 += k2 >= u ? key_value(k2) : 0.f;
    a3 += k3 >= u ? key_value(k3) : 0.f;
  }
  for (; j < nb; j += 32) {
    const uint32_t k = p[j];
    a0 += k >= u ? key_value(k) : 0.f;
  }
  return warp_sum_d((double(a0) + double(a1)) + (double(a2) + double(a3)));
}
__device__ __forceinline__ int count_at_least(const uint32_t* p, int jb, int nb, uint32_t u, int lane) {
  int c = 0;
  for (int j = jb + lane; j < nb; j += 32) c += p[j] >= u;
  return warp_sum_i(c);
}
__device__ __forceinline__ int count_equal(const uint32_t* p, int jb, int nb, uint32_t u, int lane) {
  int c = 0;
  for (int j = jb + lane; j < nb; j += 32) c += p[j] == u;
  return warp_sum_i(c);
}

// The two warps of a row each reduce their half of the row; a pair value is
// published in shared memory and combined after a 64-thread named barrier
// (one per row). Values alternate between two slots, so a slot is rewritten
// only after a later barrier that both warps passed after reading it. Both
// warps combine in the same order (half 0 + half 1): their decisions agree.
struct RowPair {
  double* xd;  // [2 slots][2 halves]
  int* xi;     // [2 slots][2 halves]
  int bar, h, lane, slot;
  __device__ __forceinline__ void sync() { named_bar_sync(bar, 64); }
  __device__ __forceinline__ double sum_d(double v) {
    if (lane == 0) xd[2 * slot + h] = v;
    sync();
    const double r = xd[2 * slot] + xd[2 * slot + 1];
    slot ^= 1;
    return r;
  }
  __device__ __forceinline__ int sum_i(int v) {
    if (lane == 0) xi[2 * slot + h] = v;
    sync();
    const int r = xi[2 * slot] + xi[2 * slot + 1];
    slot ^= 1;
    return r;
  }
  __device__ __forceinline__ float max_f(float v) {
    if (lane == 0) xd[2 * slot + h] = double(v);
    sync();
    const float r = fmaxf(float(xd[2 * slot]), float(xd[2 * slot + 1]));
    slot ^= 1;
    return r;
  }
  __device__ __forceinline__ uint32_t max_u(uint32_t v) {
    if (lane == 0) xi[2 * slot + h] = int(v);
    sync();
    const uint32_t r = max(uint32_t(xi[2 * slot]), uint32_t(xi[2 * slot + 1]));
    slot ^= 1;
    return r;
  }
  // half 0's value, for both warps
  __device__ __forceinline__ int first_i(int v) {
    if (lane == 0) xi[2 * slot + h] = v;
    sync();
    const int r = xi[2 * slot];
    slot ^= 1;
    return r;
  }
};

template <int ROWS>
__global__ void __launch_bounds__(ROWS * 64, 1)
    select_kernel(const float* __restrict__ qp, const float* __restrict__ kT, int nb, int nbp, int d, float scale,
                  const __grid_constant__ SelHeads hp, const float* __restrict__ kbias, uint32_t* __restrict__ mask,
                  int32_t* __restrict__ kept) {
  // two warps per row: all of them stream logits (more loads in flight), one per row selects
  constexpr int kThreads = ROWS * 64;
  extern __shared__ __align__(16) float sm[];
  float* srow = sm;                      // [ROWS][nb]
  float* qT = srow + size_t(ROWS) * nb;  // [d][ROWS]: one float4 = one channel of 4 rows
  const int head = blockIdx.y;
  const int I0 = blockIdx.x * ROWS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float* qh = qp + size_t(head) * nb * d;
  for (int i = tid; i < ROWS * d; i += kThreads) {
    const int r = i / d, c = i - r * d;
    qT[c * ROWS + r] = (I0 + r < nb) ? qh[size_t(I0 + r) * d + c] : 0.f;
  }
  __syncthreads();
  // ---- 1. logits. kT is the head's pooled keys transposed, [d][nbp]: for channel c a warp reads 32 x 4
  // consecutive keys (512 contiguous bytes). A thread owns keys k0 .. k0+3, k0 = 4 * (tid + i * kThreads),
  // and forms their logits against the CTA's rows (shared-memory broadcasts). Channels accumulate in
  // ascending order, one chain per (row, key).
  const float* kTh = kT + size_t(head) * d * nbp;
  for (int k0 = 4 * tid; k0 < nb; k0 += 4 * kThreads) {
    float a[ROWS][4];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) a[r][0] = a[r][1] = a[r][2] = a[r][3] = 0.f;
#pragma unroll 8
    for (int c = 0; c < d; ++c) {
      const float4 kv = __ldg(reinterpret_cast<const float4*>(kTh + size_t(c) * nbp + k0));
      const float* qc = qT + c * ROWS;
#pragma unroll
      for (int r4 = 0; r4 < ROWS / 4; ++r4) {
        const float4 qv = *reinterpret_cast<const float4*>(qc + 4 * r4);
        const float qs[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[4 * r4 + i][0] = fmaf(qs[i], kv.x, a[4 * r4 + i][0]);
          a[4 * r4 + i][1] = fmaf(qs[i], kv.y, a[4 * r4 + i][1]);
          a[4 * r4 + i][2] = fmaf(qs[i], kv.z, a[4 * r4 + i][2]);
          a[4 * r4 + i][3] = fmaf(qs[i], kv.w, a[4 * r4 + i][3]);
        }
      }
    }
#pragma unroll
    for (int jk = 0; jk < 4; ++jk) {
      const int key = k0 + jk;
      if (key < nb) {
        const float bj = kbias ? __ldg(kbias + key) : 0.f;
#pragma unroll
        for (int r = 0; r < ROWS; ++r) srow[size_t(r) * nb + key] = a[r][jk] * scale + bj;
      }
    }
  }
  __syncthreads();
  // ---- 2..5. two warps per query block, each over one half of the row
  // (split at a multiple of 32 entries, so each bitmask word has one owner)
  const int r = warp >> 1, h = warp & 1;
  const int I = I0 + r;
  if (I >= nb) return;  // both warps of the row
  RowPair pr{reinterpret_cast<double*>(qT + d * ROWS) + 4 * r, reinterpret_cast<int*>(
                 reinterpret_cast<double*>(qT + d * ROWS) + 4 * ROWS) + 4 * r, 1 + r, h, lane, 0};
  const int top_k = hp.per_head ? hp.k[head] : hp.k0;
  const float tau = hp.per_head ? hp.tau[head] : hp.tau0;
  uint32_t* p = reinterpret_cast<uint32_t*>(srow + size_t(r) * nb);
  const float* sl = srow + size_t(r) * nb;
  const int words = (nb + 31) >> 5;
  uint32_t* mrow = mask + (size_t(head) * nb + I) * words;
  const int half = ((nb + 63) >> 6) << 5;
  const int jb = h * half, je = max(jb, min(nb, jb + half));
  const int wb = jb >> 5, we = (je + 31) >> 5;  // this warp's bitmask words
  float mx = -INFINITY;
  for (int j = jb + lane; j < je; j += 32) mx = fmaxf(mx, sl[j]);  // fmaxf skips NaN
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  mx = pr.max_f(mx);
  int np = 0;
  for (int j0 = jb; j0 < je; j0 += 32) {
    const int j = j0 + lane;
    uint32_t key = 0u;
    if (j < je) {
      const float sv = sl[j];
      if (sv == sv) {  // present: NaN logits mark absent blocks
        float e = expf(sv - mx);
        if (!(e >= 0.f)) e = 0.f;  // every present logit -inf: no mass
        key = __float_as_uint(e) + 1u;
      }
      p[j] = key;
    }
    np += __popc(__ballot_sync(0xffffffffu, key != 0u));
  }
  __syncwarp();
  const int n_present = pr.sum_i(np);
  const double Z = pr.sum_d(mass_at_least(p, jb, je, 1u, lane));
  if (n_present == 0) {  // an empty query block (or no present key): empty row
    for (int w = wb + lane; w < we; w += 32) mrow[w] = 0u;
    if (h == 0 && lane == 0) kept[size_t(head) * nb + I] = 0;
    return;
  }
  if (top_k >= n_present || tau >= 1.0f) {
    // every present block
    for (int w = wb; w < we; ++w) {
      const int j = 32 * w + lane;
      const uint32_t kb = __ballot_sync(0xffffffffu, j < je && p[j] != 0u);
      if (lane == 0) mrow[w] = kb;
    }
    if (h == 0 && lane == 0) kept[size_t(head) * nb + I] = n_present;
    return;
  }
  const double target = double(tau) * Z;
  // u*: largest key with mass(key >= u) >= target.
  uint32_t u_star;
  int m_star;
  if (target <= 0.0) {
    // C_1 >= tau already: the single largest entry (ties -> lowest J).
    uint32_t best = 0;
    for (int j = jb + lane; j < je; j += 32) best = max(best, p[j]);
#pragma unroll
    for (int o = 16; o; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    u_star = pr.max_u(best);
    m_star = pr.sum_i(count_at_least(p, jb, je, u_star + 1, lane)) + 1;
  } else {
    uint32_t lo = 1, hi = 0x3F800002u;  // mass(>= lo) >= target, mass(>= hi) < target
    while (hi - lo > 1) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      if (pr.sum_d(mass_at_least(p, jb, je, mid, lane)) >= target) lo = mid; else hi = mid;
    }
    u_star = lo;
    const double above = pr.sum_d(mass_at_least(p, jb, je, u_star + 1, lane));
    const int above_cnt = pr.sum_i(count_at_least(p, jb, je, u_star + 1, lane));
    // take the entries tied at u_star in ascending J: each adds the same value
    const int ties = pr.sum_i(count_equal(p, jb, je, u_star, lane));
    double run = above;
    int rank = 0;
    bool found = false;
    for (int t = 0; t < ties && !found; ++t) {
      run += double(key_value(u_star));
      ++rank;
      found = run >= target;
    }
    if (!found) rank = max(rank, 1);
    m_star = above_cnt + rank;
  }
  const int m = max(min(top_k, n_present), m_star);
  uint32_t u_final;
  int keep_ties;  // number of entries tied at u_final to keep, lowest J first
  if (m == m_star) {
    u_final = u_star;
    keep_ties = m - pr.sum_i(count_at_least(p, jb, je, u_star + 1, lane));
  } else {
    uint32_t lo = 1, hi = 0x7F800002u;  // count(>= lo) >= m, count(>= hi) < m
    while (hi - lo > 1) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      if (pr.sum_i(count_at_least(p, jb, je, mid, lane)) >= m) lo = mid; else hi = mid;
    }
    u_final = lo;
    keep_ties = m - pr.sum_i(count_at_least(p, jb, je, u_final + 1, lane));
  }
  // ties at u_final in the first half precede those of the second
  const int ties_first = pr.first_i(count_equal(p, jb, je, u_final, lane));
  int tie_run = h == 0 ? 0 : ties_first;
  for (int w = wb; w < we; ++w) {
    const int j = 32 * w + lane;
    const uint32_t key = j < je ? p[j] : 0u;
    const bool tie = j < je && key == u_final;
    const uint32_t tb = __ballot_sync(0xffffffffu, tie);
    const int my_rank = tie_run + __popc(tb & ((1u << lane) - 1u));
    const bool keep = j < je && (key > u_final || (tie && my_rank < keep_ties));
    const uint32_t kb = __ballot_sync(0xffffffffu, keep);
    tie_run += __popc(tb);
    if (lane == 0) mrow[w] = kb;
  }
  if (h == 0 && lane == 0) kept[size_t(head) * nb + I] = m;
}

// kT[h][c][j] = kp[h][j][c] for j < nb, 0 for nb <= j < nbp (32 x 32 tiles through shared memory).
__global__ void __launch_bounds__(256) transpose_keys_kernel(const float* __restrict__ kp, int nb, int nbp, int d,
                                                             float* __restrict__ kT) {
  __shared__ float tile[32][33];
  const int h = blockIdx.z, j0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const float* src = kp + size_t(h) * nb * d;
  float* dst = kT + size_t(h) * d * nbp;
  for (int r = ty; r < 32; r += 8) {
    const int j = j0 + r, c = c0 + tx;
    tile[r][tx] = (j < nb && c < d) ? src[size_t(j) * d + c] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int c = c0 + r, j = j0 + tx;
    if (c < d && j < nbp) dst[size_t(c) * nbp + j] = tile[tx][r];
  }
}

// Exclusive scan of n ints into out[0..n] (out[n] = total), one CTA.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ in, int n, int32_t* __restrict__ out) {
  __shared__ int64_t part[1024];
  const int tid = threadIdx.x;
  const int per = (n + 1023) / 1024;
  const int b = tid * per, e = min(n, b + per);
  int64_t s = 0;
  for (int i = b; i < e; ++i) s += in[i];
  part[tid] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int64_t v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int64_t run = part[tid] - s;
  for (int i = b; i < e; ++i) {
    out[i] = int32_t(run);
    run += in[i];
  }
  if (tid == 1023) out[n] = int32_t(part[1023]);
}

__global__ void __launch_bounds__(256) fill_kernel(const uint32_t* __restrict__ mask, const int32_t* __restrict__ row_ptr,
                                                   int rows, int nb, int64_t cap, int32_t* __restrict__ col_idx,
                                                   int* status) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int words = (nb + 31) >> 5;
  const uint32_t* mrow = mask + size_t(row) * words;
  int64_t pos = row_ptr[row];
  const int64_t end = row_ptr[row + 1];
  if (end > cap || end < pos) {
    if (lane == 0) atomicOr(status, kDevErrCapacity);
    return;
  }
  for (int w0 = 0; w0 < words; w0 += 32) {
    const int w = w0 + lane;
    uint32_t bits = w < words ? mrow[w] : 0u;
    const int cnt = __popc(bits);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int64_t at = pos + incl - cnt;
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      if (at < end) col_idx[at] = 32 * w + bit;
      ++at;
    }
    pos += __shfl_sync(0xffffffffu, incl, 31);
  }
}

}  // namespace

// The status word, then the pooled keys transposed per head, [heads][d][nbp], nbp = nb rounded up to 4.
size_t block_select_ws_bytes(int heads, int nb, int d) {
  const size_t nbp = (size_t(nb) + 3) & ~size_t(3);
  return kWsHeader + align_up(size_t(heads) * d * nbp * sizeof(float), 256);
}

cudaError_t launch_exclusive_scan(const int32_t* in, int n, int32_t* out, cudaStream_t s) {
  scan_kernel<<<1, 1024, 0, s>>>(in, n, out);
  return cudaGetLastError();
}

cudaError_t launch_mask_to_lists(const uint32_t* mask, const int32_t* row_ptr, int rows, int nb, int64_t cap,
                                 int32_t* idx, int* status, cudaStream_t s) {
  fill_kernel<<<unsigned((int64_t(rows) * 32 + 255) / 256), 256, 0, s>>>(mask, row_ptr, rows, nb, cap, idx, status);
  return cudaGetLastError();
}

}  // namespace prism

using namespace prism;

namespace {

prism_status block_select_impl(const float* q_pool, const float* k_pool, int32_t heads, int32_t n_blocks,
                               int32_t head_dim, float scale, const SelHeads& hp, const float* key_bias,
                               uint32_t* mask, int32_t* kept, int32_t* row_ptr, int32_t* col_idx, int64_t col_cap,
                               int64_t* total_kept, void* ws, size_t ws_bytes, void* stream) {
  if (!q_pool || !k_pool || !mask || !kept || !row_ptr) return PRISM_ERR_ARG;
  if (heads < 1 || n_blocks < 1) return PRISM_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return PRISM_ERR_ARG;
  if (head_dim != 64 && head_dim != 128) return PRISM_ERR_UNSUPPORTED;
  if (n_blocks > kSelMaxBlocks) return PRISM_ERR_UNSUPPORTED;
  if (int64_t(heads) * n_blocks * n_blocks >= (int64_t(1) << 31)) return PRISM_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(q_pool) % 16 || reinterpret_cast<uintptr_t>(k_pool) % 16) return PRISM_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(key_bias) % 4) return PRISM_ERR_ARG;
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < block_select_ws_bytes(heads, n_blocks, head_dim))
    return PRISM_ERR_WORKSPACE;
  if (col_idx && col_cap < 0) return PRISM_ERR_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int nbp = (n_blocks + 3) & ~3;
  float* kT = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kWsHeader);
  transpose_keys_kernel<<<dim3((nbp + 31) / 32, (head_dim + 31) / 32, heads), 256, 0, s>>>(k_pool, n_blocks, nbp,
                                                                                        head_dim, kT);
  const int rows_per_cta = n_blocks <= kSelMaxBlocks8 ? 8 : 4;
  // logits [rows][nb], query rows [d][rows], then the row pairs' exchange slots (4 doubles + 4 ints per row)
  const size_t smem = (size_t(rows_per_cta) * n_blocks + size_t(head_dim) * rows_per_cta) * sizeof(float) +
                      size_t(rows_per_cta) * (4 * sizeof(double) + 4 * sizeof(int));
  const dim3 grid((n_blocks + rows_per_cta - 1) / rows_per_cta, heads);
  if (rows_per_cta == 8) {
    if (cudaFuncSetAttribute(select_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
      return PRISM_ERR_CUDA;
    select_kernel<8><<<grid, 512, smem, s>>>(q_pool, kT, n_blocks, nbp, head_dim, scale, hp, key_bias, mask, kept);
  } else {
    if (cudaFuncSetAttribute(select_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
      return PRISM_ERR_CUDA;
    select_kernel<4><<<grid, 256, smem, s>>>(q_pool, kT, n_blocks, nbp, head_dim, scale, hp, key_bias, mask, kept);
  }
  const int rows = heads * n_blocks;
  if (launch_exclusive_scan(kept, rows, row_ptr, s) != cudaSuccess) return PRISM_ERR_CUDA;
  if (total_kept) {
    int32_t tot = 0;
    if (cudaMemcpyAsync(&tot, row_ptr + rows, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return PRISM_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PRISM_ERR_CUDA;
    *total_kept = tot;
    if (col_idx && tot > col_cap) return PRISM_ERR_CAPACITY;
  }
  if (col_idx) {
    if (launch_mask_to_lists(mask, row_ptr, rows, n_blocks, col_cap, col_idx, ws_status(ws), s) != cudaSuccess)
      return PRISM_ERR_CUDA;
  }
  return cuda_status(cudaGetLastError());
}

}  // namespace

extern "C" prism_status prism_block_select(const float* q_pool, const float* k_pool, int32_t heads, int32_t n_blocks,
                                           int32_t head_dim, float scale, int32_t top_k, float cdf_threshold,
                                           uint32_t* mask, int32_t* kept, int32_t* row_ptr, int32_t* col_idx,
                                           int64_t col_cap, int64_t* total_kept, void* ws, size_t ws_bytes,
                                           void* stream) {
  if (top_k < 1 || !(cdf_threshold >= 0.f)) return PRISM_ERR_ARG;
  SelHeads hp{};
  hp.per_head = 0;
  hp.k0 = top_k;
  hp.tau0 = cdf_threshold;
  return block_select_impl(q_pool, k_pool, heads, n_blocks, head_dim, scale, hp, nullptr, mask, kept, row_ptr,
                           col_idx, col_cap, total_kept, ws, ws_bytes, stream);
}

extern "C" prism_status prism_block_select_ex(const float* q_pool, const float* k_pool, int32_t heads,
                                              int32_t n_blocks, int32_t head_dim, float scale,
                                              const prism_select_params* params, uint32_t* mask, int32_t* kept,
                                              int32_t* row_ptr, int32_t* col_idx, int64_t col_cap,
                                              int64_t* total_kept, void* ws, size_t ws_bytes, void* stream) {
  if (!params || heads < 1) return PRISM_ERR_ARG;
  SelHeads hp{};
  hp.k0 = params->top_k;
  hp.tau0 = params->cdf_threshold;
  const bool per_head = params->head_top_k || params->head_cdf_threshold;
  if (per_head) {
    if (heads > kSelMaxHeads) return PRISM_ERR_UNSUPPORTED;
    hp.per_head = 1;
    for (int h = 0; h < heads; ++h) {
      hp.k[h] = params->head_top_k ? params->head_top_k[h] : params->top_k;
      hp.tau[h] = params->head_cdf_threshold ? params->head_cdf_threshold[h] : params->cdf_threshold;
      if (hp.k[h] < 1 || !(hp.tau[h] >= 0.f)) return PRISM_ERR_ARG;
    }
  } else if (hp.k0 < 1 || !(hp.tau0 >= 0.f)) {
    return PRISM_ERR_ARG;
  }
  return block_select_impl(q_pool, k_pool, heads, n_blocks, head_dim, scale, hp, params->key_bias, mask, kept,
                           row_ptr, col_idx, col_cap, total_kept, ws, ws_bytes, stream);
}

extern "C" prism_status prism_block_select_workspace_size(int32_t heads, int32_t n_blocks, int32_t head_dim,
                                                          size_t* bytes) {
  if (!bytes || heads < 1 || n_blocks < 1 || head_dim < 1) return PRISM_ERR_ARG;
  *bytes = block_select_ws_bytes(heads, n_blocks, head_dim);
  return PRISM_OK;
}

extern "C" prism_status prism_topk_from_sparsity(float sparsity, int32_t n_blocks, int32_t* top_k) {
  if (!top_k || n_blocks < 1 || !(sparsity >= 0.f) || !(sparsity < 1.f)) return PRISM_ERR_ARG;
  const int64_t dropped = int64_t(std::floor(double(sparsity) * double(n_blocks)));
  *top_k = int32_t(std::max<int64_t>(1, int64_t(n_blocks) - dropped));
  return PRISM_OK;
}

extern "C" prism_status prism_mask_to_csr(const uint32_t* mask, const int32_t* row_ptr, int32_t rows,
                                          int32_t n_blocks, int32_t* col_idx, int64_t col_cap, void* ws,
                                          size_t ws_bytes, void* stream) {
  if (!mask || !row_ptr || !col_idx || rows < 1 || n_blocks < 1 || col_cap < 0) return PRISM_ERR_ARG;
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < kWsHeader) return PRISM_ERR_WORKSPACE;
  return cuda_status(launch_mask_to_lists(mask, row_ptr, rows, n_blocks, col_cap, col_idx, ws_status(ws),
                                          reinterpret_cast<cudaStream_t>(stream)));
}
