// a4 + a5: block scoring and hybrid top-k + cumulative-mass selection.
//
// Prism walkthrough (wmrh.cn/news/72296), section "三者如何协同": the gating
// step keeps the k highest-scoring blocks, then extends along the CDF of the
// block scores until cdf_threshold (default 0.20). Prism README "Overview":
// the hybrid rule sets each query's sparsity. Sol-Attn abstract on the Prism
// paper page: blocks are ranked by a block proxy score.
//
// Three kernels per call, the last two once per chunk of heads:
//   split_tf32_kernel: q_pool and k_pool into tf32-exact halves, x = hi + lo
//     (hi keeps the top 10 mantissa bits of x, lo = x - hi is exact in fp32).
//   score_kernel: the logits s_IJ = scale * qbar_I . kbar_J (+ b_J, the
//     optional key-block bias, walkthrough section "桥接残差反哺稀疏注意力") of
//     a chunk of heads as a tcgen05 kind::tf32 GEMM in split precision:
//     hi.hi + hi.lo + lo.hi accumulated in fp32 in tensor memory (relative
//     error about 2^-20 of sum_c |q_c k_c|, against 2^-8 for one bf16 product).
//     A persistent CTA per SM takes 128 x 256 tiles in turn: the 32-channel
//     slices of the four operand halves come by TMA (128-byte swizzle) into a
//     two-stage ring, two TMEM accumulators let the epilogue of one tile
//     overlap the products of the next, and the logits leave as 32 x 32 TMA
//     box stores (128-byte rows) into the workspace, a round of heads at a
//     time (up to 1 GiB of logits; one head of the 2K grid is 85 MB).
//   select_rows_kernel: one 128-thread CTA per (head, query block), the row's
//     entries in registers (thread t holds J = t + 128 i):
//     1. max of the present logits (a NaN logit marks an absent block: an
//        empty block of a grid clipped at its edge), p_J = exp(s_J - max),
//        Z = sum p (fp32 chains of at most VPT terms per thread, combined in
//        fp64 in a fixed order);
//     2. the mass threshold u* = max{u : sum_{p_J >= u} p_J >= tau Z}: a
//        bisection on the float bits of p inside the row's [min, max] bracket
//        until at most 32 entries remain in the bracket (or one value); those
//        are sorted in one warp and their masses added in rank order in fp64;
//        the count m* follows, ties at u* taken in ascending J;
//     3. m = max(k, m*); when k decides, the same bracketed search on counts
//        finds the k-th largest entry;
//     4. the kept set (p descending, ties to the lower J) written as bitmask
//        words by warp ballots, and kept[row] = m.
//   k and tau are the row's head's (per-head settings, walkthrough section
//   "实际案例与上手参考": the top-k part of the selection is a tunable ratio).
// scan_kernel: exclusive scan of kept into the CSR row_ptr (one CTA).
// fill_kernel: one warp per row expands the bitmask into ascending col_idx.
#include <algorithm>
#include <cfloat>
#include <cmath>

#include "host.h"
#include "ptx.cuh"

namespace prism {
namespace {

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

// ------------------------------------------------------------------ split
// hi = x with the low 13 mantissa bits cleared (exactly a tf32 value, so the
// tensor core reads it unchanged); lo = x - hi, exact in fp32, of which the
// tensor core keeps the top 10 mantissa bits. NaN stays NaN in both.
__global__ void __launch_bounds__(256) split_tf32_kernel(const float4* __restrict__ x, size_t n4,
                                                         float4* __restrict__ hi, float4* __restrict__ lo) {
  for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n4; i += size_t(gridDim.x) * blockDim.x) {
    const float4 v = x[i];
    float4 h, l;
    h.x = __uint_as_float(__float_as_uint(v.x) & 0xFFFFE000u);
    h.y = __uint_as_float(__float_as_uint(v.y) & 0xFFFFE000u);
    h.z = __uint_as_float(__float_as_uint(v.z) & 0xFFFFE000u);
    h.w = __uint_as_float(__float_as_uint(v.w) & 0xFFFFE000u);
    l.x = v.x - h.x;
    l.y = v.y - h.y;
    l.z = v.z - h.z;
    l.w = v.w - h.w;
    hi[i] = h;
    lo[i] = l;
  }
}

// ------------------------------------------------------------------ scores
constexpr int kScM = 128;                      // query blocks per tile (TMEM lanes)
constexpr int kScN = 256;                      // key blocks per tile (TMEM columns)
constexpr int kScAtomBytes = 128;              // 32 fp32 channels: one 128-byte swizzle row
constexpr int kScABytes = kScM * kScAtomBytes;  // 16 KB
constexpr int kScBBytes = kScN * kScAtomBytes;  // 32 KB
constexpr int kScStageBytes = 2 * kScABytes + 2 * kScBBytes;  // A hi, A lo, B hi, B lo
constexpr int kScStages = 2;
constexpr int kScEpiWarps = 4;
constexpr int kScStageOut = 32 * 128;  // one epilogue store tile: 32 rows x 32 logits
constexpr int kScOutOff = kScStages * kScStageBytes;
constexpr int kScBarOff = kScOutOff + kScEpiWarps * 2 * kScStageOut;
constexpr int kScSmem = kScBarOff + 256 + 1024;  // + barriers, + alignment slack
constexpr int kScThreads = 64 + 32 * kScEpiWarps;

struct ScoreParams {
  CUtensorMap q_hi, q_lo, k_hi, k_lo;  // 3-D fp32 (d, n_blocks, heads), box (32, 128 | 256, 1)
  CUtensorMap out;                     // logits, 3-D fp32 (nbp, n_blocks, round heads), box (32, 32, 1)
  const float* kbias;                  // [nb] or null
  int nb, d, head0, heads;             // heads: in this round
  float scale;
  int* status;
};

// Instruction descriptor for kind::tf32 with fp32 accumulation, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// 3-D tiled store from this CTA's shared memory (bulk-group completion); box
// elements outside the tensor are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
// Waits until at most one committed bulk store of this thread still reads its source.
__device__ __forceinline__ void bulk_wait_group_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
// Waits until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Persistent: CTA b takes tiles b, b + grid, ... of the round; tile t is
// (head t / (rows * cols), query tile, key tile) in raster order.
//   warp 0      copies: per 32-channel slice, A hi/lo (128 query blocks) and
//               B hi/lo (256 key blocks) into a two-stage ring;
//   warp 1      TMEM owner and MMA issuer: per slice 4 x (lo.hi, hi.lo, hi.hi)
//               products into one of two 256-column accumulators;
//   warps 2..5  epilogue: a thread per TMEM lane (query block), 32 logits per
//               load, scaled (+ bias), through a swizzled shared-memory tile
//               into one 32 x 32 TMA box store (128-byte rows);
// the epilogue of tile i overlaps the products of tile i + 1.
__global__ void __launch_bounds__(kScThreads, 1) score_kernel(const __grid_constant__ ScoreParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kScBarOff);
  uint64_t* full = bars;            // [2] slice landed
  uint64_t* empty = bars + 2;       // [2] slice's products complete
  uint64_t* acc_full = bars + 4;    // [2] accumulator's products complete
  uint64_t* acc_empty = bars + 6;   // [2] accumulator read by the epilogue warps
  uint64_t* mma_done = bars + 8;    // every product complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 10);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int atoms = P.d / 32;
  const int n_it = (P.nb + kScM - 1) / kScM, n_jt = (P.nb + kScN - 1) / kScN;
  const int total = P.heads * n_it * n_jt;
  int* status = P.status;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kScStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kScEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kScN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&P.q_hi);
      tma_prefetch_desc(&P.q_lo);
      tma_prefetch_desc(&P.k_hi);
      tma_prefetch_desc(&P.k_lo);
      bool ok = true;
      int it = 0;  // slices issued
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const int hz = t / (n_it * n_jt), r = t - hz * n_it * n_jt;
        const int I0 = (r / n_jt) * kScM, J0 = (r % n_jt) * kScN, head = P.head0 + hz;
        for (int a = 0; a < atoms; ++a) {
          const int st = it % kScStages;
          // stage st last held slice it - 2: free once its products completed
          if (it >= kScStages) ok = mbar_wait_abortable(&empty[st], ((it / kScStages) - 1) & 1, status, abort_flag);
          if (!ok) break;
          uint8_t* sb = sm + st * kScStageBytes;
          mbar_arrive_expect_tx(&full[st], kScStageBytes);
          tma_load_3d(sb, &P.q_hi, &full[st], 32 * a, I0, head);
          tma_load_3d(sb + kScABytes, &P.q_lo, &full[st], 32 * a, I0, head);
          tma_load_3d(sb + 2 * kScABytes, &P.k_hi, &full[st], 32 * a, J0, head);
          tma_load_3d(sb + 2 * kScABytes + kScBBytes, &P.k_lo, &full[st], 32 * a, J0, head);
          ++it;
        }
      }
      // drain: every issued copy has landed before the CTA may exit
      for (int i = it - kScStages > 0 ? it - kScStages : 0; i < it; ++i)
        mbar_wait(&full[i % kScStages], (i / kScStages) & 1, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_tf32_f32(kScM, kScN);
      bool ok = true;
      int it = 0, lt = 0;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++lt) {
        const int acc = lt & 1;
        // accumulator acc last held tile lt - 2: free once the epilogue read it
        if (lt >= 2) ok = mbar_wait_abortable(&acc_empty[acc], ((lt >> 1) - 1) & 1, status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d = tbase + acc * kScN;
        for (int a = 0; a < atoms && ok; ++a) {
          const int st = it % kScStages;
          ok = mbar_wait_abortable(&full[st], (it / kScStages) & 1, status, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sb = smem_u32(sm + st * kScStageBytes);
          const uint64_t ahi = sdesc_sw128(sb, 16, 1024), alo = sdesc_sw128(sb + kScABytes, 16, 1024);
          const uint64_t bhi = sdesc_sw128(sb + 2 * kScABytes, 16, 1024);
          const uint64_t blo = sdesc_sw128(sb + 2 * kScABytes + kScBBytes, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 8 tf32 channels (32 bytes) per product
            const uint64_t o = uint64_t(kk * 2);
            mma_tf32(d, alo + o, bhi + o, idesc, (a > 0 || kk > 0) ? 1u : 0u);
            mma_tf32(d, ahi + o, blo + o, idesc, 1u);
            mma_tf32(d, ahi + o, bhi + o, idesc, 1u);
          }
          mma_commit(&empty[st]);
          ++it;
        }
        if (ok) mma_commit(&acc_full[acc]);
      }
      // every product this thread issued has completed before TMEM is released
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    uint8_t* outb = sm + kScOutOff + (warp - 2) * 2 * kScStageOut;
    int sbuf = 0, lt = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++lt) {
      const int hz = t / (n_it * n_jt), r = t - hz * n_it * n_jt;
      const int I0 = (r / n_jt) * kScM, J0 = (r % n_jt) * kScN;
      const int acc = lt & 1;
      if (!mbar_wait_abortable(&acc_full[acc], (lt >> 1) & 1, status, abort_flag)) break;
      tc_fence_after();
      const bool rows_in = I0 + 32 * q < P.nb;  // some of this warp's query blocks exist
#pragma unroll 1
      for (int c = 0; c < kScN / 32; ++c) {
        const int Jc = J0 + 32 * c;
        if (Jc >= P.nb || !rows_in) break;  // warp-uniform
        uint32_t rr[32];
        tmem_ld32(tbase + acc * kScN + lane_off + 32 * c, rr);
        tmem_ld_wait();
        // the store tile written two stores ago has been read
        if (lane == 0) bulk_wait_group_read1();
        __syncwarp();
        uint8_t* tile = outb + sbuf * kScStageOut;
#pragma unroll
        for (int qq = 0; qq < 8; ++qq) {
          float v[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int J = Jc + 4 * qq + e;
            const float b = (P.kbias && J < P.nb) ? __ldg(P.kbias + J) : 0.f;
            v[e] = __uint_as_float(rr[4 * qq + e]) * P.scale + b;
          }
          *reinterpret_cast<float4*>(tile + sw128_offset(lane, qq)) = make_float4(v[0], v[1], v[2], v[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&P.out, tile, Jc, I0 + 32 * q, hz);
          bulk_commit_group();
        }
        sbuf ^= 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
    }
    if (lane == 0) bulk_wait_group0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 2 * kScN);
  }
}

// ------------------------------------------------------------------ selection
constexpr int kSelThreads = 128;  // threads per row
constexpr int kSelWarps = kSelThreads / 32;

// Per-warp partial results in shared memory; two slots alternate, so a slot
// is rewritten only after a later barrier that every warp passed after reading it.
struct SelShared {
  double d[2][kSelWarps];
  int i[2][kSelWarps];
  uint32_t u[2][kSelWarps][2];
  float f[2][kSelWarps];
  float lp[32];      // the entries of a final bracket (at most 32), in no order
  float sorted[32];  // the same, descending
  int lcount;
  int res_i[4];
  uint32_t res_u[2];
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

// Sum over the CTA of (fp64 mass, int count); every thread gets the same
// result (partials combined in warp order).
__device__ __forceinline__ void cta_sum(double& m, int& c, SelShared& S, int& slot, int warp, int lane) {
  m = warp_sum_d(m);
  c = warp_sum_i(c);
  if (lane == 0) {
    S.d[slot][warp] = m;
    S.i[slot][warp] = c;
  }
  __syncthreads();
  m = (S.d[slot][0] + S.d[slot][1]) + (S.d[slot][2] + S.d[slot][3]);
  c = (S.i[slot][0] + S.i[slot][1]) + (S.i[slot][2] + S.i[slot][3]);
  slot ^= 1;
}

// Mass (fp32 chain per thread, fp64 across threads) and count of the entries >= pm.
template <int VPT>
__device__ __forceinline__ void mass_count_at_least(const float (&p)[VPT], float pm, double& m, int& c) {
  float a = 0.f;
  int n = 0;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    if (p[i] >= pm) {  // false for NaN (absent); a compare and two predicated adds per entry
      a += p[i];
      ++n;
    }
  }
  m = a;
  c = n;
}

// Gathers the entries of [lo, hi) (at most 32) into S.lp, then warp 0 sorts
// them descending and picks the entry that decides the search: in mass mode
// the first, in rank order, whose running mass (from mass_hi, fp64) reaches
// the target; in count mode the one of rank need - cnt_hi - 1. Publishes its
// value, the count of entries above it and the count of entries equal to it.
template <int VPT>
__device__ __forceinline__ void resolve_bracket(const float (&p)[VPT], uint32_t lo, uint32_t hi, int cnt_hi,
                                             double mass_hi, bool mass_mode, double target, int need,
                                             SelShared& S) {
  if (threadIdx.x == 0) S.lcount = 0;
  __syncthreads();
  const float plo = __uint_as_float(lo), phi = __uint_as_float(hi);
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    if (p[i] >= plo && p[i] < phi) {
      const int at = atomicAdd(&S.lcount, 1);
      if (at < 32) S.lp[at] = p[i];
    }
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int c = min(S.lcount, 32);
    const float v = lane < c ? S.lp[lane] : -1.f;
    int rank = 0;  // descending; equal values take consecutive ranks in list order
    for (int o = 0; o < c; ++o) {
      const float w = S.lp[o];
      rank += (w > v) || (w == v && o < lane);
    }
    if (lane < c) S.sorted[rank] = v;
    __syncwarp();
    const float vr = lane < c ? S.sorted[lane] : -1.f;
    int pick;
    if (mass_mode) {
      double cum = lane < c ? double(vr) : 0.0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double t = __shfl_up_sync(0xffffffffu, cum, o);
        if (lane >= o) cum += t;
      }
      cum += mass_hi;
      const uint32_t reach = __ballot_sync(0xffffffffu, lane < c && cum >= target);
      pick = reach ? __ffs(reach) - 1 : c - 1;
      if (lane == 0) S.res_i[1] = cnt_hi + pick + 1;  // the count up to the decisive entry
    } else {
      pick = need - cnt_hi - 1;
    }
    const float u = __shfl_sync(0xffffffffu, vr, pick);
    const uint32_t above = __ballot_sync(0xffffffffu, lane < c && vr > u);
    const uint32_t equal = __ballot_sync(0xffffffffu, lane < c && vr == u);
    if (lane == 0) {
      S.res_u[0] = __float_as_uint(u);
      S.res_i[0] = cnt_hi + __popc(above);
      S.res_i[2] = __popc(equal);
    }
  }
  __syncthreads();
}

template <int VPT>
__global__ void __launch_bounds__(kSelThreads) select_rows_kernel(const float* __restrict__ logits, int nb, int nbp,
                                                                  int head0, const __grid_constant__ SelHeads hp,
                                                                  uint32_t* __restrict__ mask,
                                                                  int32_t* __restrict__ kept) {
  __shared__ SelShared S;
  __shared__ int tie_cnt[VPT][kSelWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hz = blockIdx.x / nb, I = blockIdx.x - hz * nb;
  const int head = head0 + hz;
  const int words = (nb + 31) >> 5;
  uint32_t* mrow = mask + (size_t(head) * nb + I) * words;
  int32_t* krow = kept + size_t(head) * nb + I;
  const float* srow = logits + size_t(blockIdx.x) * nbp;
  int slot = 0;
  // ---- 1. logits, maximum, p = exp(s - max) (as 2^((s - max) log2 e))
  float p[VPT];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int J = tid + kSelThreads * i;
    p[i] = J < nb ? __ldg(srow + J) : __uint_as_float(0x7fc00000u);
    mx = fmaxf(mx, p[i]);  // fmaxf skips NaN
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) S.f[slot][warp] = mx;
  __syncthreads();
  mx = fmaxf(fmaxf(S.f[slot][0], S.f[slot][1]), fmaxf(S.f[slot][2], S.f[slot][3]));
  slot ^= 1;
  const float mx2 = mx * 1.44269504088896341f;
  uint32_t umin = 0xFFFFFFFFu, umax = 0u;
  int np = 0;
  float zs = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    if (p[i] == p[i]) {  // present
      // hardware 2^x (relative error about 2^-22, far below the mass comparisons' margin)
      float e;
      asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(fmaf(p[i], 1.44269504088896341f, -mx2)));
      if (!(e >= 0.f)) e = 0.f;  // every present logit -inf: no mass
      e = fminf(e, 1.f);
      p[i] = e;
      umin = min(umin, __float_as_uint(e));
      umax = max(umax, __float_as_uint(e));
      zs += e;
      ++np;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    umin = min(umin, __shfl_xor_sync(0xffffffffu, umin, o));
    umax = max(umax, __shfl_xor_sync(0xffffffffu, umax, o));
  }
  if (lane == 0) {
    S.u[slot][warp][0] = umin;
    S.u[slot][warp][1] = umax;
  }
  double Z = zs;
  cta_sum(Z, np, S, slot, warp, lane);  // its barrier also publishes the minima and maxima
  const int sl = slot ^ 1;
  umin = min(min(S.u[sl][0][0], S.u[sl][1][0]), min(S.u[sl][2][0], S.u[sl][3][0]));
  umax = max(max(S.u[sl][0][1], S.u[sl][1][1]), max(S.u[sl][2][1], S.u[sl][3][1]));
  const int top_k = hp.per_head ? hp.k[head] : hp.k0;
  const float tau = hp.per_head ? hp.tau[head] : hp.tau0;
  if (np == 0 || top_k >= np || tau >= 1.0f) {
    // an empty query block (or no present key): empty row; else every present block
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const uint32_t b = __ballot_sync(0xffffffffu, np > 0 && p[i] == p[i]);
      const int w = i * kSelWarps + warp;
      if (lane == 0 && w < words) mrow[w] = b;
    }
    if (tid == 0) *krow = np;
    return;
  }
  const double target = double(tau) * Z;
  // ---- 2. the mass threshold, then 3. the floor k, with one bracketed search:
  // mass mode keeps mass(>= lo) >= target > mass(>= hi); count mode keeps
  // count(>= lo) >= m > count(>= hi). Each pass halves [lo, hi) in float bits;
  // the search ends at one value or at most 32 entries in the bracket.
  uint32_t lo = umin, hi = umax + 1u;
  int cnt_lo = np, cnt_hi = 0;
  double mass_hi = 0.0;
  bool mass_mode = true;
  int need = 0, m = 0;
  uint32_t u_final = 0;
  int cnt_gt = 0, ties_total = 0;  // entries above u_final, entries equal to it
  if (target <= 0.0) lo = umax;  // the first entry in rank order reaches the target already
#pragma unroll 1
  for (int round = 0; round < 2; ++round) {
    if (round == 1) {
      // the floor decides: the m-th largest entry lies at or below u*
      mass_mode = false;
      need = m;
      lo = umin;
      hi = u_final + 1u;
      cnt_lo = np;
      cnt_hi = cnt_gt;
    } else if (target <= 0.0) {
      double ms;
      int c;
      mass_count_at_least(p, __uint_as_float(lo), ms, c);
      cta_sum(ms, c, S, slot, warp, lane);
      cnt_lo = c;
    }
#pragma unroll 1
    while (cnt_lo - cnt_hi > 32 && hi - lo > 1u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      double ms;
      int c;
      mass_count_at_least(p, __uint_as_float(mid), ms, c);
      cta_sum(ms, c, S, slot, warp, lane);
      if (mass_mode ? (ms >= target) : (c >= need)) {
        lo = mid;
        cnt_lo = c;
      } else {
        hi = mid;
        cnt_hi = c;
        mass_hi = ms;
      }
    }
    int m_here;
    if (hi - lo == 1u) {
      // one value left: tied entries, each adding the same mass
      u_final = lo;
      cnt_gt = cnt_hi;
      ties_total = cnt_lo - cnt_hi;
      if (mass_mode) {
        const double pv = double(__uint_as_float(lo));
        double run = mass_hi;
        int r = 0;
        while (r < ties_total) {
          run += pv;
          ++r;
          if (run >= target) break;
        }
        m_here = cnt_hi + max(r, 1);
      } else {
        m_here = need;
      }
    } else {
      resolve_bracket(p, lo, hi, cnt_hi, mass_hi, mass_mode, target, need, S);
      u_final = S.res_u[0];
      cnt_gt = S.res_i[0];
      ties_total = S.res_i[2];
      m_here = mass_mode ? S.res_i[1] : need;
    }
    if (round == 0) {
      m = max(min(top_k, np), m_here);
      if (m == m_here) break;  // the mass decides
    }
  }
  const int keep_ties = m - cnt_gt;
  // ---- 4. bitmask: p > u_final, and the first keep_ties entries equal to u_final in ascending J
  // (J = 128 i + 32 warp + lane: slot-major, then warp, then lane)
  const float uf = __uint_as_float(u_final);
  if (keep_ties >= ties_total) {
    // every entry equal to u_final is kept
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const uint32_t kb = __ballot_sync(0xffffffffu, p[i] >= uf);
      const int w = i * kSelWarps + warp;
      if (lane == 0 && w < words) mrow[w] = kb;
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const uint32_t tb = __ballot_sync(0xffffffffu, p[i] == uf);
      if (lane == 0) tie_cnt[i][warp] = __popc(tb);
    }
    __syncthreads();
    int run = 0;  // ties before the current slot
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      int before = run;
      for (int w = 0; w < warp; ++w) before += tie_cnt[i][w];
      run += (tie_cnt[i][0] + tie_cnt[i][1]) + (tie_cnt[i][2] + tie_cnt[i][3]);
      const bool tie = p[i] == uf;
      const uint32_t tb = __ballot_sync(0xffffffffu, tie);
      const int my_rank = before + __popc(tb & ((1u << lane) - 1u));
      const bool keep = p[i] > uf || (tie && my_rank < keep_ties);
      const uint32_t kb = __ballot_sync(0xffffffffu, keep);
      const int w = i * kSelWarps + warp;
      if (lane == 0 && w < words) mrow[w] = kb;
    }
  }
  if (tid == 0) *krow = m;
}

// Exclusive scan of n ints into out[0..n] (out[n] = total), one CTA: thread t owns a contiguous chunk
// (a multiple of four entries), summed and rewritten with 16-byte accesses when both buffers are
// 16-byte aligned, so its loads are in flight together instead of one dependent load per entry.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ in, int n, int32_t* __restrict__ out) {
  __shared__ int64_t part[1024];
  const int tid = threadIdx.x;
  const int per = (((n + 1023) / 1024) + 3) & ~3;
  const int b = min(n, tid * per), e = min(n, b + per);
  const bool vec = ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 15u) == 0;
  const int ev = vec ? b + ((e - b) & ~3) : b;  // [b, ev) in int4 steps, then [ev, e) one by one
  int64_t s = 0;
#pragma unroll 4
  for (int i = b; i < ev; i += 4) {
    const int4 v = *reinterpret_cast<const int4*>(in + i);
    s += int64_t(v.x) + v.y + v.z + v.w;
  }
  for (int i = ev; i < e; ++i) s += in[i];
  part[tid] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const int64_t v = tid >= off ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  int64_t run = part[tid] - s;
#pragma unroll 2
  for (int i = b; i < ev; i += 4) {
    const int4 v = *reinterpret_cast<const int4*>(in + i);
    int4 o;
    o.x = int32_t(run);
    run += v.x;
    o.y = int32_t(run);
    run += v.y;
    o.z = int32_t(run);
    run += v.z;
    o.w = int32_t(run);
    run += v.w;
    *reinterpret_cast<int4*>(out + i) = o;
  }
  for (int i = ev; i < e; ++i) {
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

// Entries per thread of select_rows_kernel: n_blocks / 128 rounded up to an instantiated size.
constexpr int kVpts[] = {1, 2, 4, 8, 12, 16, 24, 32, 36, 40, 48, 64, 80};

int select_vpt(int nb) {
  const int need = (nb + kSelThreads - 1) / kSelThreads;
  for (int v : kVpts)
    if (v >= need) return v;
  return 0;
}

template <int V>
cudaError_t launch_rows_v(const float* logits, int nb, int nbp, int h0, int g, const SelHeads& hp, uint32_t* mask,
                          int32_t* kept, cudaStream_t s) {
  select_rows_kernel<V><<<unsigned(g) * unsigned(nb), kSelThreads, 0, s>>>(logits, nb, nbp, h0, hp, mask, kept);
  return cudaGetLastError();
}

cudaError_t launch_select_rows(int vpt, const float* logits, int nb, int nbp, int h0, int g, const SelHeads& hp,
                               uint32_t* mask, int32_t* kept, cudaStream_t s) {
  switch (vpt) {
#define PRISM_ROWS_CASE(V) \
  case V: return launch_rows_v<V>(logits, nb, nbp, h0, g, hp, mask, kept, s);
    PRISM_ROWS_CASE(1) PRISM_ROWS_CASE(2) PRISM_ROWS_CASE(4) PRISM_ROWS_CASE(8) PRISM_ROWS_CASE(12)
    PRISM_ROWS_CASE(16) PRISM_ROWS_CASE(24) PRISM_ROWS_CASE(32) PRISM_ROWS_CASE(36) PRISM_ROWS_CASE(40)
    PRISM_ROWS_CASE(48) PRISM_ROWS_CASE(64) PRISM_ROWS_CASE(80)
#undef PRISM_ROWS_CASE
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// Heads whose logits one score/selection round holds: as many as fit in 1 GiB, at least one. A round
// is one persistent score launch and one row launch over all its heads; at 2K (85 MB of logits per
// head) rounds of one head cost 0.6 ms more over 24 heads in launch gaps and tails than rounds of 12.
#ifndef PRISM_SELECT_ROUND_MIB
#define PRISM_SELECT_ROUND_MIB 1024
#endif
int select_chunk_heads(int heads, int nb) {
  const size_t nbp = (size_t(nb) + 3) & ~size_t(3);
  const size_t per_head = size_t(nb) * nbp * sizeof(float);
  const size_t budget = size_t(PRISM_SELECT_ROUND_MIB) << 20;
  return int(std::max<size_t>(1, std::min<size_t>(size_t(heads), budget / per_head)));
}

// The status word, then the tf32 halves of the pooled features (q hi, q lo, k hi, k lo, each
// [heads][nb][d] fp32), then one round's logits [chunk heads][nb][nbp], nbp = nb rounded up to 4.
size_t block_select_ws_bytes(int heads, int nb, int d) {
  const size_t nbp = (size_t(nb) + 3) & ~size_t(3);
  const size_t half = align_up(size_t(heads) * nb * d * sizeof(float), 256);
  return kWsHeader + 4 * half + align_up(size_t(select_chunk_heads(heads, nb)) * nb * nbp * sizeof(float), 256);
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
  const size_t n_el = size_t(heads) * n_blocks * head_dim;
  const size_t half = align_up(n_el * sizeof(float), 256);
  uint8_t* base = static_cast<uint8_t*>(ws) + kWsHeader;
  float* q_hi = reinterpret_cast<float*>(base);
  float* q_lo = reinterpret_cast<float*>(base + half);
  float* k_hi = reinterpret_cast<float*>(base + 2 * half);
  float* k_lo = reinterpret_cast<float*>(base + 3 * half);
  float* logits = reinterpret_cast<float*>(base + 4 * half);
  {
    const size_t n4 = n_el / 4;
    const unsigned blocks = unsigned(std::min<size_t>((n4 + 255) / 256, size_t(device_sm_count()) * 16));
    split_tf32_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(q_pool), n4,
                                             reinterpret_cast<float4*>(q_hi), reinterpret_cast<float4*>(q_lo));
    split_tf32_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(k_pool), n4,
                                             reinterpret_cast<float4*>(k_hi), reinterpret_cast<float4*>(k_lo));
  }
  const int chunk = select_chunk_heads(heads, n_blocks);
  ScoreParams sp;
  {
    const uint64_t dims[3] = {uint64_t(head_dim), uint64_t(n_blocks), uint64_t(heads)};
    const uint64_t strides[2] = {uint64_t(head_dim) * 4, uint64_t(n_blocks) * head_dim * 4};
    const uint32_t box_a[3] = {32, kScM, 1}, box_b[3] = {32, kScN, 1};
    const uint64_t odims[3] = {uint64_t(nbp), uint64_t(n_blocks), uint64_t(chunk)};
    const uint64_t ostrides[2] = {uint64_t(nbp) * 4, uint64_t(n_blocks) * nbp * 4};
    const uint32_t box_o[3] = {32, 32, 1};
    prism_status st = PRISM_OK;
    if ((st = encode_tiled(&sp.q_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, q_hi, dims, strides, box_a,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != PRISM_OK ||
        (st = encode_tiled(&sp.q_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, q_lo, dims, strides, box_a,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != PRISM_OK ||
        (st = encode_tiled(&sp.k_hi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, k_hi, dims, strides, box_b,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != PRISM_OK ||
        (st = encode_tiled(&sp.k_lo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, k_lo, dims, strides, box_b,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != PRISM_OK ||
        (st = encode_tiled(&sp.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, logits, odims, ostrides, box_o,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != PRISM_OK)
      return st;
  }
  sp.kbias = key_bias;
  sp.nb = n_blocks;
  sp.d = head_dim;
  sp.scale = scale;
  sp.status = ws_status(ws);
  if (cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kScSmem) != cudaSuccess)
    return PRISM_ERR_CUDA;
  const int vpt = select_vpt(n_blocks);
  const int tiles_per_head = ((n_blocks + kScM - 1) / kScM) * ((n_blocks + kScN - 1) / kScN);
  for (int h0 = 0; h0 < heads; h0 += chunk) {
    const int g = std::min(chunk, heads - h0);
    sp.head0 = h0;
    sp.heads = g;
    const int grid = std::min(g * tiles_per_head, device_sm_count());
    score_kernel<<<grid, kScThreads, kScSmem, s>>>(sp);
    if (launch_select_rows(vpt, logits, n_blocks, nbp, h0, g, hp, mask, kept, s) != cudaSuccess)
      return PRISM_ERR_CUDA;
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
