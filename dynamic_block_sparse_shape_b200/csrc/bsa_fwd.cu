// a6: block-sparse attention forward over the selected blocks.
//
// Sol-Attn abstract on the Prism paper page: dynamic sparse attention computes
// only the selected key/value blocks. Prism README, "Overview": the selection
// is per query block (hybrid rule). The attention over the selection is
// exact: an online softmax over the kept 64-token key blocks (FlashAttention
// style), fp32 statistics and accumulators, bf16 operands.
//
// One CTA per (query block I, head); a step covers two selected key blocks.
// Warp roles:
//   warp 0      copy producer: Q once, through a 5-D tensor map (one per
//               block shape); per step K and V of the step's two key blocks
//               (3-slot rings each) as bulk copies of their block images
//               (written by block_images_kernel before the attention kernel);
//   warp 1      TMEM owner and issuer of the score products
//               S_j = Q [K_j0 K_j1]^T  (.ws M=64, N=128, K=d, Q from TMEM);
//   warps 2..9  softmax, two groups of four warps taking alternate steps
//               (group j % 2 takes step j), one thread per TMEM lane: a
//               thread holds the 64 scores of one query row against one key
//               block of the step;
//   warp 10     issuer of the value products
//               O_g += P_j [V_j0 | V_j1]  (.ws M=64, N=2d, K=64, P from TMEM).
// Two issuing threads feed the one tensor pipe: while one waits on a barrier
// the other's products keep the pipe busy. Two softmax groups keep each SM
// sub-partition busy: while one group waits (barriers, tensor-memory loads),
// the other computes exponentials.
// TMEM holds every tensor-core A operand: Q, and P (one buffer per group).
// The .ws datapath computes the accumulator columns n < N/2 in lanes 0..63
// from A rows in lanes 0..63 and the columns n >= N/2 in lanes 64..127 from
// A rows in lanes 64..127. S_j of key block 0 lands in the low lanes and of
// key block 1 in the high lanes, so the P rows each lane half holds belong to
// one key block, and the value product takes its B operand's first d columns
// from V of key block 0 and the next d from V of key block 1: lane m
// accumulates the block-0 part of O row m, lane m + 64 the block-1 part, over
// all d channels. Each group has its own O parts, so every (group, lane half)
// part keeps its own running max and sum: no thread exchanges a row maximum
// with another while the row is streamed. The four parts of a row are merged
// once, in the epilogue. P never touches shared memory, so per step shared
// memory carries only the K and V tiles (bulk-copy writes, tensor-core reads).
// The producer never blocks on one barrier: it polls the barriers of every
// copy it could start next (mbarrier.test_wait) and starts whichever is
// ready. Each issuer waits for its own operands in step order. K slot j%3 is
// refilled once S_j has completed, V slot j%3 once PV_j has; a group's S
// buffer once its warps have read it, its P buffer once its last PV has
// completed.
// A part's running max is only moved when it grows by more than 8 (log2
// units); the final merge uses the same stale maxima, so the result is exact
// while the rare O rescale (TMEM load/scale/store) stays off the common path.
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "bsa_common.cuh"
#include "host.h"

namespace prism {
namespace {

constexpr int kKB = 2;      // key blocks per step
constexpr int kRing = 3;    // K slots = V slots
constexpr int kGroups = 2;  // softmax warp groups, alternate steps
constexpr int kGroupWarps = 4;
constexpr int kSoftWarps = kGroups * kGroupWarps;
constexpr int kFwdThreads = 64 + 32 * kSoftWarps + 32;
constexpr int kPvWarp = 2 + kSoftWarps;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kSmallSteps = 4;  // rows of up to 8 key blocks go to bsa_fwd_small_kernel

struct FwdParams {
  CUtensorMap mq[kMaxCand];
  CUtensorMap mo[kMaxCand];   // O and its rounding residual, for bf16 outputs:
  CUtensorMap mol[kMaxCand];  // the epilogue stores a block's rows with 5-D box copies
  CUtensorMap mk[kMaxCand];   // K and V, for the short-row kernel when it takes every row
  CUtensorMap mv[kMaxCand];
  const uint8_t* kimg;  // block images of K and V (layout in host.h)
  const uint8_t* vimg;
  Geo g;
  const int32_t* zone_shape;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  void* o;
  float* lse;
  __nv_bfloat16* o_lo;  // rounding residual of a bf16 o, or null
  int* status;
  int64_t tok_stride;  // of o, elements
  float scale_log2;
  int out_fp32;
  int tma_out;  // bf16 output: stores through the O / o_lo tensor maps
  int heads;
  int all_rows;  // the short-row kernel takes every row, K and V through mk / mv (no block images)
};

template <int D>
struct FwdSmem {
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kQBytes = D * 128;
  static constexpr uint32_t kSlotBytes = kKB * D * 128;      // K (or V) of one step
  static constexpr uint32_t kK0 = kQBytes;                   // [slot][dh][block][64][128 B]
  static constexpr uint32_t kV0 = kK0 + kRing * kSlotBytes;  // [slot][block][dh][64][128 B]
  static constexpr uint32_t kRed = kV0 + kRing * kSlotBytes; // per part: running max, sum [4][64] each
  static constexpr uint32_t kRedBytes = 2 * 4 * 64 * 4;
  static constexpr uint32_t kDesc = kRed + kRedBytes;  // block-id ring
  static constexpr uint32_t kBar = kDesc + kDescRing * 4;
  static constexpr uint32_t kTotal = kBar + 256;
  // epilogue exchange of merged O quarters: [lane half][group][64 rows][D/4 + 4 floats], over the K ring
  static constexpr uint32_t kXPitch = D / 4 + 4;
  static_assert(4 * 64 * kXPitch * 4 <= kRing * kSlotBytes, "exchange buffer fits the K ring");
  // TMEM: S buffers (64 columns per group) at 0; O parts (D columns per
  // group) at 128; Q (A operand, D/2 columns); P buffers (32 columns per group)
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kTO = 64 * kGroups;
  static constexpr uint32_t kTQ = kTO + kGroups * D;
  static constexpr uint32_t kTP = kTQ + D / 2;
  static_assert(kTP + kGroups * 32 <= kTmemCols, "TMEM budget");
};

// Maximum of 64 scores (raw bits of fp32 values).
__device__ __forceinline__ float max64(const uint32_t* r) {
  float ca = fmax3(__uint_as_float(r[0]), __uint_as_float(r[1]), __uint_as_float(r[2]));
  float cb = fmax3(__uint_as_float(r[3]), __uint_as_float(r[4]), __uint_as_float(r[5]));
#pragma unroll
  for (int i = 6; i < 62; i += 4) {
    ca = fmax3(ca, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
    cb = fmax3(cb, __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
  }
  return fmax3(fmaxf(ca, cb), __uint_as_float(r[62]), __uint_as_float(r[63]));
}

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1) bsa_fwd_kernel(const __grid_constant__ FwdParams P) {
  using L = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;    // [3] K of the slot's step landed
  uint64_t* v_full = bars + 4;    // [3] V of the slot's step landed
  uint64_t* k_free = bars + 7;    // [3] S of the slot's step complete
  uint64_t* v_free = bars + 10;   // [3] PV of the slot's step complete
  uint64_t* s_full = bars + 13;   // [2] per group: its current S complete
  uint64_t* s_free = bars + 15;   // [2] per group: its S read by its 4 warps
  uint64_t* p_full = bars + 17;   // [2] per group: its P written to TMEM by its 4 warps
  uint64_t* p_free = bars + 19;   // [2] per group: its PV complete (P buffer and O parts quiescent)
  uint64_t* mma_done = bars + 21;
  uint64_t* pv_done = bars + 22;
  uint64_t* qa_full = bars + 23;  // Q copied into TMEM by the softmax warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 25);
  float* redm = reinterpret_cast<float*>(sm + L::kRed);
  float* redl = redm + 4 * 64;

  const Geo& g = P.g;
  const int I = blockIdx.x, head = blockIdx.y;
  const int row = head * g.n_blocks + I;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = P.status;
  const int beg = P.row_ptr[row];
  int cnt = P.row_ptr[row + 1] - beg;
  if (cnt < 0 || cnt > g.n_blocks) {
    if (threadIdx.x == 0) atomicOr(status, kDevErrBounds);
    cnt = 0;
  }
  const int nsteps = (cnt + kKB - 1) / kKB;
  if (nsteps <= kSmallSteps) return;  // short and empty rows: bsa_fwd_small_kernel's

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&k_free[i], 1);
      mbar_init(&v_free[i], 1);
    }
    for (int i = 0; i < kGroups; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kGroupWarps);
      mbar_init(&p_full[i], kGroupWarps);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(pv_done, 1);
    mbar_init(qa_full, kSoftWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t tO = tbase + L::kTO;
  const uint32_t tQ = tbase + L::kTQ;
  const uint32_t tP = tbase + L::kTP;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (nsteps > 0) {
      IdCache dc{reinterpret_cast<int*>(sm + L::kDesc), 0};
      if (lane == 0) {
        const int sI = safe_shape(g, P.zone_shape, I, status);
        const BlockBox qb = block_box(g, sI, I);
        mbar_arrive_expect_tx(q_full, L::kQBytes);
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_5d(sm + L::kQ + dh * kBoxBytes, &P.mq[sI], q_full, dh * 64, head, qb.w0, qb.h0, qb.t0);
      }
      int kj = 0, vj = 0;
#ifdef PRISM_FAULT_INJECTION
      // test builds only: when the workspace word after the status word is set, the CTA of
      // (query block 0, head 0) never issues the K copies of its second step, so the score
      // issuer's bounded wait for them runs out (the timeout path under test)
      const int skip_k = (blockIdx.x == 0 && blockIdx.y == 0 &&
                          *reinterpret_cast<volatile int*>(status + 1) != 0) ? 1 : -1;
#endif
      Watchdog wd;
      wd.reset();
      while (kj < nsteps || vj < nsteps) {
        if (kj < nsteps) dc.ensure(kKB * kj + kKB - 1, g, P.col_idx, beg, cnt, status, lane);
        int nk = kj, nv = vj, stop = 0;
        if (lane == 0) {
          bool did = false;
          // K slot nk%3 last held the K of step nk-3: free once S_{nk-3} completed
          if (nk < nsteps && mbar_test(&k_free[nk % kRing], ((nk / kRing) & 1) ^ 1)) {
            const int ks = nk % kRing;
            bool issue = true;
#ifdef PRISM_FAULT_INJECTION
            issue = nk != skip_k;
#endif
            if (issue) {
              uint8_t* dst = sm + L::kK0 + ks * L::kSlotBytes;
              mbar_arrive_expect_tx(&k_full[ks], L::kSlotBytes);
              for (int slot = 0; slot < kKB; ++slot) {
                const uint8_t* src = P.kimg + image_offset(g, head, dc.get(kKB * nk + slot), D);
                for (int dh = 0; dh < D / 64; ++dh)
                  bulk_load(dst + dh * (kKB * kBoxBytes) + slot * kBoxBytes, src + dh * kBoxBytes, kBoxBytes,
                            &k_full[ks]);
              }
            }
            ++nk;
            did = true;
          }
          // V slot nv%3 last held the V of step nv-3: free once PV_{nv-3} completed
          if (nv < nk && mbar_test(&v_free[nv % kRing], ((nv / kRing) & 1) ^ 1)) {
            const int vs = nv % kRing;
            uint8_t* dst = sm + L::kV0 + vs * L::kSlotBytes;
            mbar_arrive_expect_tx(&v_full[vs], L::kSlotBytes);
            for (int slot = 0; slot < kKB; ++slot)
              bulk_load(dst + slot * (D * 128), P.vimg + image_offset(g, head, dc.get(kKB * nv + slot), D), D * 128,
                        &v_full[vs]);
            ++nv;
            did = true;
          }
          if (did) wd.reset();
          else if (!wd.ok(status, abort_flag)) stop = 1;
        }
        kj = __shfl_sync(0xffffffffu, nk, 0);
        vj = __shfl_sync(0xffffffffu, nv, 0);
        if (__shfl_sync(0xffffffffu, stop, 0)) break;
      }
      if (lane == 0) {
        // drain: every issued copy has landed before the CTA may exit
        mbar_wait(q_full, 0, status);
        for (int i = kj - kRing > 0 ? kj - kRing : 0; i < kj; ++i)
          mbar_wait(&k_full[i % kRing], (i / kRing) & 1, status);
        for (int i = vj - kRing > 0 ? vj - kRing : 0; i < vj; ++i)
          mbar_wait(&v_full[i % kRing], (i / kRing) & 1, status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ score issuer
    if (lane == 0 && nsteps > 0) {
      const uint32_t idS = idesc_bf16_f32(64, 64 * kKB, false, false);
      const uint64_t dK0 = sdesc_sw128(smem_u32(sm + L::kK0), 16, 1024);
      bool ok = mbar_wait_abortable(qa_full, 0, status, abort_flag);
      for (int sj = 0; sj < nsteps && ok; ++sj) {
        const int b = sj % kRing, gs = sj & 1;
        // K of step sj landed; the group's S buffer read by its warps (its previous step)
        ok = mbar_wait_abortable(&k_full[b], (sj / kRing) & 1, status, abort_flag) &&
             mbar_wait_abortable(&s_free[gs], ((sj >> 1) & 1) ^ 1, status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dK = dK0 + uint64_t(b * (L::kSlotBytes >> 4));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ws_ts(tbase + gs * 64, tQ + kk * 8, dK + kmajor_step(kk, kKB * kBoxBytes), idS, kk > 0 ? 1u : 0u);
        mma_commit(&s_full[gs]);
        mma_commit(&k_free[b]);
      }
      // every product this thread issued has completed before TMEM is released
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, status);
    }
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ value issuer
    if (lane == 0 && nsteps > 0) {
      // B = V of the step, MN-major, N = 2d: the d channels of key block 0
      // (64-column chunks kBoxBytes apart, as the slot holds [block][dh]),
      // then those of key block 1. One product per 16-key step.
      const uint32_t idO = idesc_bf16_f32(64, 2 * D, false, true);
      const uint64_t dV0 = sdesc_sw128(smem_u32(sm + L::kV0), kBoxBytes, 1024);
      bool ok = true;
      for (int pj = 0; pj < nsteps && ok; ++pj) {
        const int b = pj % kRing, gp = pj & 1;
        ok = mbar_wait_abortable(&p_full[gp], (pj >> 1) & 1, status, abort_flag) &&
             mbar_wait_abortable(&v_full[b], (pj / kRing) & 1, status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t dV = dV0 + uint64_t(b * (L::kSlotBytes >> 4));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ws_ts(tO + gp * D, tP + gp * 32 + kk * 8, dV + uint64_t((kk * 2048) >> 4), idO,
                    (pj >= kGroups || kk > 0) ? 1u : 0u);
        mma_commit(&p_free[gp]);
        mma_commit(&v_free[b]);
      }
      mma_commit(pv_done);
      mbar_wait(pv_done, 0, status);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 2;
    const int grp = sw / kGroupWarps;
    const int sp = warp & 3;  // TMEM lane quarter of this warp
    const int Ln = sp * 32 + lane;
    const int m = Ln & 63, kh = Ln >> 6;
    const int part = grp * 2 + kh;  // warp-uniform
    const uint32_t lane_off = uint32_t(sp * 32) << 16;
    float m_run = -INFINITY, l_part = 0.f;
    if (nsteps > 0) {
      // Q becomes the A operand of every S product: one copy into TMEM
      // (the two groups copy the two column halves)
      mbar_wait_abortable(q_full, 0, status, abort_flag);
      tile_to_tmem_a<D>(sm + L::kQ, tQ + lane_off, m, grp);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qa_full);
    }
    int k = 0;  // this group's step count
    for (int j = grp; j < nsteps; j += kGroups, ++k) {
      const bool valid = (j * kKB + kh) < cnt;  // warp-uniform: kh is fixed per warp
      // keys of a key block clipped by the grid's edge (read before the wait)
      uint64_t members = ~uint64_t(0);
      if (g.partial && valid) members = key_block_members(g, P.zone_shape, __ldg(P.col_idx + beg + j * kKB + kh));
      mbar_wait_abortable(&s_full[grp], k & 1, status, abort_flag);
      tc_fence_after();
      uint32_t r[64];
      tmem_ld32(tbase + lane_off + grp * 64, r);
      tmem_ld32(tbase + lane_off + grp * 64 + 32, r + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[grp]);
      mask_scores32(r, uint32_t(members));
      mask_scores32(r + 32, uint32_t(members >> 32));
      // the scale is positive, so it commutes with the max
      const float mx = valid ? max64(r) * P.scale_log2 : -INFINITY;
      const float m_new = fmaxf(m_run, mx);
      const bool resc = m_new > m_run + kRescaleThreshold;
      if (__any_sync(0xffffffffu, resc)) {
        const float alpha = resc ? fast_exp2(m_run - m_new) : 1.f;
        if (resc) {
          l_part *= alpha;
          m_run = m_new;
        }
        if (k > 0) {
          // this lane's O part holds the group's earlier PVs: wait for the last, then rescale
          mbar_wait_abortable(&p_free[grp], (k - 1) & 1, status, abort_flag);
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < D / 32; ++h) {
            uint32_t o[32];
            const uint32_t ta = tO + grp * D + lane_off + h * 32;
            tmem_ld32(ta, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(ta, o);
            tmem_st16(ta + 16, o + 16);
          }
          tmem_st_wait();
        }
      }
      uint32_t pk[32];
      if (valid) {
        // m_run is finite unless every key so far lay outside the grid (then every p is 0)
        const float c = P.scale_log2, nm = m_run == -INFINITY ? 0.f : -m_run;
        float la = 0.f, lb = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(r[2 * i]), c, nm));
          const float p1 = fast_exp2(fmaf(__uint_as_float(r[2 * i + 1]), c, nm));
          la += p0;
          lb += p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        l_part += la + lb;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
      }
      // the group's P buffer: free once its previous PV completed
      if (k > 0) mbar_wait_abortable(&p_free[grp], (k - 1) & 1, status, abort_flag);
      tmem_st16(tP + lane_off + grp * 32, pk);
      tmem_st16(tP + lane_off + grp * 32 + 16, pk + 16);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[grp]);
    }
    // ---------------------------------------------------------- epilogue
    // k = this group's step count; its last PV complete before O is read
    if (k > 0) mbar_wait_abortable(&p_free[grp], (k - 1) & 1, status, abort_flag);
    tc_fence_after();
    redm[part * 64 + m] = m_run;
    redl[part * 64 + m] = l_part;
    named_bar_sync(1, 32 * kSoftWarps);
    const bool ok = *abort_flag == 0;  // uniform: read after the barrier
    // merge the row's four parts: max M, sum L = sum_p l_p 2^(m_p - M)
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < 4; ++q) M = fmaxf(M, redm[q * 64 + m]);
    float Lsum = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lq = redl[q * 64 + m];
      if (lq > 0.f) Lsum += lq * fast_exp2(redm[q * 64 + m] - M);
    }
    const float inv = (Lsum > 0.f && ok) ? 1.f / Lsum : 0.f;
    // weights of the two groups' parts held in this thread's TMEM lane (the
    // key-block-kh half of row m); a group that took no step has no O part
    float wg[kGroups];
#pragma unroll
    for (int gq = 0; gq < kGroups; ++gq) {
      const int q = gq * 2 + kh;
      wg[gq] = redl[q * 64 + m] > 0.f ? fast_exp2(redm[q * 64 + m] - M) * inv : 0.f;
    }
    const int sI = safe_shape(g, P.zone_shape, I, status);
    const BlockBox qb = block_box(g, sI, I);
    const int tok = block_token(g, qb, m);
    // a query slot outside the grid (a block clipped by the edge) has no output
    const bool row_in = !g.partial || block_slot_in_grid(g, qb, m);
    // This thread merges both groups' parts of its lane over channel half grp,
    // keeps quarter grp * 2 + kh of the row and hands quarter grp * 2 + (kh ^ 1)
    // to the thread of the other lane half (same group, same row).
    constexpr int NC = D / 4;
    const int keep = grp * (D / 2) + kh * NC, give = grp * (D / 2) + (kh ^ 1) * NC;
    float* X = reinterpret_cast<float*>(sm + L::kK0);
    float ov[NC], gv[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) ov[i] = gv[i] = 0.f;
#pragma unroll
    for (int gq = 0; gq < kGroups; ++gq) {
      if (nsteps > gq) {  // CTA-uniform: group gq took at least one step
        float a[NC], b[NC];
        tmem_ld_f<NC>(tO + gq * D + lane_off + keep, a);
        tmem_ld_f<NC>(tO + gq * D + lane_off + give, b);
        const float w = wg[gq];
#pragma unroll
        for (int i = 0; i < NC; ++i) {
          ov[i] = fmaf(a[i], w, ov[i]);
          gv[i] = fmaf(b[i], w, gv[i]);
        }
      }
    }
    float* xo = X + ((kh * 2 + grp) * 64 + m) * L::kXPitch;
#pragma unroll
    for (int i = 0; i < NC / 4; ++i)
      reinterpret_cast<float4*>(xo)[i] = make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]);
    named_bar_sync(1, 32 * kSoftWarps);
    const float* xi = X + (((kh ^ 1) * 2 + grp) * 64 + m) * L::kXPitch;
#pragma unroll
    for (int i = 0; i < NC / 4; ++i) {
      const float4 t = reinterpret_cast<const float4*>(xi)[i];
      ov[4 * i] += t.x;
      ov[4 * i + 1] += t.y;
      ov[4 * i + 2] += t.z;
      ov[4 * i + 3] += t.w;
    }
    // o[i] keeps 0 where every weight is 0 (no key, or an abort)
#pragma unroll
    for (int i = 0; i < NC; ++i) ov[i] = inv == 0.f ? 0.f : ov[i];
    if (P.tma_out) {
      // bf16 rows of the block into two swizzled [d/64][64][128 B] tiles in
      // the V ring (free: every product is complete), then one box store per
      // 64 channels; rows outside the grid fall outside the tensor and are
      // not written
      uint8_t* to = sm + L::kV0;
      uint8_t* tl = to + D * 128;
      const int dh = keep / 64, c0 = (keep % 64) / 8;
#pragma unroll
      for (int q = 0; q < NC / 8; ++q) {
        float lo[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) lo[i] = ov[8 * q + i] - __bfloat162float(__float2bfloat16_rn(ov[8 * q + i]));
        const uint32_t so = dh * kBoxBytes + sw128_offset(m, c0 + q);
        *reinterpret_cast<uint4*>(to + so) =
            make_uint4(pack_bf16x2(ov[8 * q], ov[8 * q + 1]), pack_bf16x2(ov[8 * q + 2], ov[8 * q + 3]),
                       pack_bf16x2(ov[8 * q + 4], ov[8 * q + 5]), pack_bf16x2(ov[8 * q + 6], ov[8 * q + 7]));
        *reinterpret_cast<uint4*>(tl + so) =
            make_uint4(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]), pack_bf16x2(lo[4], lo[5]),
                       pack_bf16x2(lo[6], lo[7]));
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 32 * kSoftWarps);
      if (warp == 2 && lane == 0) {
        for (int h = 0; h < D / 64; ++h) {
          tma_store_5d(&P.mo[sI], to + h * kBoxBytes, h * 64, head, qb.w0, qb.h0, qb.t0);
          if (P.o_lo) tma_store_5d(&P.mol[sI], tl + h * kBoxBytes, h * 64, head, qb.w0, qb.h0, qb.t0);
        }
        bulk_commit_group();
        bulk_wait_group_read0();  // the tiles stay valid until read
      }
    } else {
      const int64_t off = int64_t(tok) * P.tok_stride + int64_t(head) * D + keep;
      if (row_in) store_row<NC>(P.o, off, ov, P.out_fp32);
      if (P.o_lo && row_in) {
        // what the bf16 store of O dropped: O = o + o_lo to about 16 bits
        float lo[NC];
#pragma unroll
        for (int i = 0; i < NC; ++i) lo[i] = ov[i] - __bfloat162float(__float2bfloat16_rn(ov[i]));
        store_row<NC>(P.o_lo, off, lo, false);
      }
    }
    if (part == 0 && row_in) {
      const int N = g.T * g.H * g.W;
      P.lse[int64_t(head) * N + tok] = (Lsum > 0.f && ok) ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, L::kTmemCols);
  }
}

// ---------------------------------------------------------------- short rows
// Rows of at most kSmallSteps steps (and empty rows) go to a second kernel
// whose CTA needs half of the tensor memory and about 100 KB of shared
// memory, so two CTAs share an SM. A row of a few key blocks is mostly fixed
// cost: copy latencies and the epilogue. Each CTA loops over the rows of its
// stride and pipelines them: the copies of the next row (its Q, then its first
// K and V) start as soon as the current row frees their buffers, and the next
// row's first score product runs while the softmax warps finish the current
// row's epilogue. Long rows stay with bsa_fwd_kernel, which returns at once
// for the short ones. With `all_rows` set (the host's plan when the rows are
// short on average) this kernel takes every row and gathers K and V through
// 5-D tensor maps: no block images are made and bsa_fwd_kernel is not
// launched.
//   warp 0      copies: per row Q (5-D TMA) into one staging tile, free again
//               once the softmax warps have moved Q into TMEM; per step K and
//               V of the step's two key blocks into one K and one V slot;
//   warp 1      TMEM owner, issues S_j = Q [K_j0 K_j1]^T and then
//               O += P_j [V_j0 | V_j1] (.ws M=64; Q and P from TMEM), one
//               step at a time: P_j is written over S_j's first 32 columns,
//               so S_{j+1} waits for PV_j, and a row's first PV waits until
//               the epilogue has read the previous row's O;
//   warps 2..5  softmax, one thread per TMEM lane (row m of the block,
//               key-block half kh of the step), running max and sum per
//               lane half, merged in the epilogue; between a row's last step
//               and its epilogue they move the next row's Q into TMEM.
// Barrier phases run on across rows: the copies, products and arrivals of the
// CTA's s-th step complete phase s of their barriers, and the row barriers
// (Q staged, Q in TMEM, O read) count the CTA's rows with work. Every wait is
// placed so that the phase after the awaited one needs a step the waiter has
// not yet enabled.
constexpr int kSmallThreads = 64 + 128;

template <int D>
struct FwdSmallSmem {
  static constexpr uint32_t kQ = 0;                      // [dh][64][128 B]
  static constexpr uint32_t kQBytes = D * 128;
  static constexpr uint32_t kSlotBytes = kKB * D * 128;  // K (or V) of one step
  static constexpr uint32_t kK = kQBytes;                // [dh][block][64][128 B]
  static constexpr uint32_t kV = kK + kSlotBytes;        // [block][dh][64][128 B]
  static constexpr uint32_t kRed = kV + kSlotBytes;      // per lane half: running max, sum [2][64] each
  static constexpr uint32_t kRedBytes = 2 * 2 * 64 * 4;
  // epilogue exchange of half rows in rounds of kXC channels, [lane half][64 rows][kXC + 4 floats];
  // then the staging tile of a bf16 output block ([dh][64][128 B], swizzled) for its box stores
  static constexpr int kXC = 32;
  static constexpr uint32_t kXPitch = kXC + 4;
  static constexpr uint32_t kX = kRed + kRedBytes;
  static constexpr uint32_t kXBytes = 2 * 64 * kXPitch * 4;
  static_assert(kX % 1024 == 0 && kXBytes >= D * 128, "the exchange buffer holds one swizzled output tile");
  static constexpr uint32_t kDesc = kX + kXBytes;  // block-id ring
  static constexpr uint32_t kBar = kDesc + kDescRing * 4;
  static constexpr uint32_t kTotal = kBar + 128;
  static_assert(2 * (kTotal + 2048) <= 228 * 1024, "two CTAs per SM");
  // TMEM: S (P over its first 32 columns) at 0, the O parts at 64 (D columns), Q at 64 + D (D/2)
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kTO = 64;
  static constexpr uint32_t kTQ = 64 + D;
  static_assert(kTQ + D / 2 <= kTmemCols, "TMEM budget");
};

// Output rows of an empty query block: O = 0 (and its residual), LSE = -inf.
// tid: 0..127.
template <int D>
__device__ __forceinline__ void write_empty_row(const FwdParams& P, int I, int head, int tid) {
  const Geo& g = P.g;
  const int m = tid & 63, half = tid >> 6;
  int* status = P.status;
  const int sI = safe_shape(g, P.zone_shape, I, status);
  const BlockBox qb = block_box(g, sI, I);
  if (g.partial && !block_slot_in_grid(g, qb, m)) return;
  const int tok = block_token(g, qb, m);
  constexpr int NC = D / 2;
  float z[NC];
#pragma unroll
  for (int i = 0; i < NC; ++i) z[i] = 0.f;
  const int64_t off = int64_t(tok) * P.tok_stride + int64_t(head) * D + half * NC;
  store_row<NC>(P.o, off, z, P.out_fp32);
  if (P.o_lo) store_row<NC>(P.o_lo, off, z, false);
  if (half == 0) P.lse[int64_t(head) * g.T * g.H * g.W + tok] = -INFINITY;
}

// List of row `row`: its first entry and its length (a malformed length is
// reported and read as 0).
__device__ __forceinline__ int row_list(const FwdParams& P, int row, int* beg) {
  const int b = __ldg(P.row_ptr + row);
  int cnt = __ldg(P.row_ptr + row + 1) - b;
  if (cnt < 0 || cnt > P.g.n_blocks) {
    atomicOr(P.status, kDevErrBounds);
    cnt = 0;
  }
  *beg = b;
  return cnt;
}

// Whether the short-row kernel computes a row of `nsteps` > 0 steps.
__device__ __forceinline__ bool small_takes(const FwdParams& P, int nsteps) {
  return P.all_rows || nsteps <= kSmallSteps;
}

// Copies one key block's K (or V) tile for the short-row kernel: from its block
// image, or (all_rows) through the 5-D tensor map of its shape, from the box
// origin {shape, t0, h0, w0} cached with its id. K tiles are laid out
// [dh][block][64][128 B] (dst = slot base), V tiles [block][dh][64][128 B].
template <int D>
__device__ __forceinline__ void small_load_kv(const FwdParams& P, bool is_v, uint8_t* slot, int kb_slot, int head,
                                              int J, int4 box, uint64_t* bar) {
  const Geo& g = P.g;
  if (P.all_rows) {
    const CUtensorMap* map = is_v ? &P.mv[box.x] : &P.mk[box.x];
    for (int dh = 0; dh < D / 64; ++dh) {
      const uint32_t off = is_v ? kb_slot * (D * 128) + dh * kBoxBytes : dh * (kKB * kBoxBytes) + kb_slot * kBoxBytes;
      tma_load_5d(slot + off, map, bar, dh * 64, head, box.w, box.z, box.y);
    }
  } else {
    const uint8_t* src = (is_v ? P.vimg : P.kimg) + image_offset(g, head, J, D);
    if (is_v) {
      bulk_load(slot + kb_slot * (D * 128), src, D * 128, bar);
    } else {
      for (int dh = 0; dh < D / 64; ++dh)
        bulk_load(slot + dh * (kKB * kBoxBytes) + kb_slot * kBoxBytes, src + dh * kBoxBytes, kBoxBytes, bar);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kSmallThreads, 2) bsa_fwd_small_kernel(const __grid_constant__ FwdParams P) {
  using L = FwdSmallSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* q_full = bars + 0;   // Q of the row staged
  uint64_t* qa_full = bars + 1;  // Q of the row in TMEM, staging tile free (4 warps)
  uint64_t* k_full = bars + 2;   // K of the step landed
  uint64_t* k_free = bars + 3;   // S of the step complete (K slot free)
  uint64_t* v_full = bars + 4;   // V of the step landed
  uint64_t* s_full = bars + 5;   // S of the step complete
  uint64_t* p_full = bars + 6;   // P of the step written (4 warps)
  uint64_t* pv_done = bars + 7;  // PV of the step complete (V slot and S / P columns free)
  uint64_t* o_free = bars + 8;   // O of the row read by the epilogue (4 warps)
  uint64_t* mma_done = bars + 9;
  uint64_t* stage_free = bars + 10;  // the rounding-residual tile of the row, staged over Q, read
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 12);
  float* redm = reinterpret_cast<float*>(sm + L::kRed);
  float* redl = redm + 2 * 64;
  float* X = reinterpret_cast<float*>(sm + L::kX);
  const Geo& g = P.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = P.status;
  const int rows = P.heads * g.n_blocks;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 11; ++i) mbar_init(&bars[i], (i == 1 || i == 6 || i == 8) ? 4 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t tO = tbase + L::kTO, tQ = tbase + L::kTQ;

  // CTA b takes rows b, b + grid, ... (row = head * n_blocks + query block);
  // every role walks the same sequence and skips the same rows
  // bf16 output with a rounding residual: the residual tile is staged over the Q tile
  const bool stage_lo = P.tma_out && P.o_lo;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    IdCache dc{reinterpret_cast<int*>(sm + L::kDesc), 0};
    if (P.all_rows) dc.zone_shape = P.zone_shape;
    bool ok = true;
    int lq = 0, gs = 0, q_iss = 0, k_iss = 0, v_iss = 0;
    for (int row = blockIdx.x; row < rows && ok; row += gridDim.x) {
      int beg;
      const int cnt = row_list(P, row, &beg);
      const int nsteps = (cnt + kKB - 1) / kKB;
      if (nsteps == 0 || !small_takes(P, nsteps)) continue;
      const int I = row % g.n_blocks, head = row / g.n_blocks;
      if (lane == 0) {
        // the staging tile held the previous row's Q until it reached TMEM,
        // then (bf16 output with a residual) the rounding residual of row lq - 2
        // until its box stores read it
        if (lq > 0) ok = mbar_wait_abortable(qa_full, (lq - 1) & 1, status, abort_flag);
        if (ok && lq > 1 && stage_lo)
          ok = mbar_wait_abortable(stage_free, (lq - 2) & 1, status, abort_flag);
        if (ok) {
          const int sI = safe_shape(g, P.zone_shape, I, status);
          const BlockBox qb = block_box(g, sI, I);
          mbar_arrive_expect_tx(q_full, L::kQBytes);
          for (int dh = 0; dh < D / 64; ++dh)
            tma_load_5d(sm + L::kQ + dh * kBoxBytes, &P.mq[sI], q_full, dh * 64, head, qb.w0, qb.h0, qb.t0);
          q_iss = lq + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      dc.filled = 0;
      for (int j = 0; j < nsteps && ok; ++j, ++gs) {
        dc.ensure(kKB * j + kKB - 1, g, P.col_idx, beg, cnt, status, lane);
        int4 bx[kKB] = {};
        if (P.all_rows)
          for (int slot = 0; slot < kKB; ++slot) bx[slot] = dc.box(kKB * j + slot);
        if (lane == 0) {
          // the K slot last held step gs - 1: free once its S completed
          if (gs > 0) ok = mbar_wait_abortable(k_free, (gs - 1) & 1, status, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(k_full, L::kSlotBytes);
            for (int slot = 0; slot < kKB; ++slot)
              small_load_kv<D>(P, false, sm + L::kK, slot, head, dc.get(kKB * j + slot), bx[slot], k_full);
            k_iss = gs + 1;
          }
          // the V slot last held step gs - 1: free once its PV completed
          if (ok && gs > 0) ok = mbar_wait_abortable(pv_done, (gs - 1) & 1, status, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(v_full, L::kSlotBytes);
            for (int slot = 0; slot < kKB; ++slot)
              small_load_kv<D>(P, true, sm + L::kV, slot, head, dc.get(kKB * j + slot), bx[slot], v_full);
            v_iss = gs + 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      ++lq;
    }
    if (lane == 0) {
      // drain: every issued copy has landed before the CTA may exit (one buffer each: the last)
      if (q_iss > 0) mbar_wait(q_full, (q_iss - 1) & 1, status);
      if (k_iss > 0) mbar_wait(k_full, (k_iss - 1) & 1, status);
      if (v_iss > 0) mbar_wait(v_full, (v_iss - 1) & 1, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(64, 64 * kKB, false, false);
      const uint64_t dK = sdesc_sw128(smem_u32(sm + L::kK), 16, 1024);
      // B = V of the step, MN-major, N = 2d: the d channels of key block 0, then those of key block 1
      const uint32_t idO = idesc_bf16_f32(64, 2 * D, false, true);
      const uint64_t dV = sdesc_sw128(smem_u32(sm + L::kV), kBoxBytes, 1024);
      bool ok = true;
      int lq = 0, gs = 0;
      for (int row = blockIdx.x; row < rows && ok; row += gridDim.x) {
        int beg;
        const int cnt = row_list(P, row, &beg);
        const int nsteps = (cnt + kKB - 1) / kKB;
        if (nsteps == 0 || !small_takes(P, nsteps)) continue;
        // Q of the row in TMEM
        ok = mbar_wait_abortable(qa_full, lq & 1, status, abort_flag);
        for (int j = 0; j < nsteps && ok; ++j, ++gs) {
          // K of the step landed; PV of the previous step (which read P from the S columns) complete
          ok = mbar_wait_abortable(k_full, gs & 1, status, abort_flag) &&
               (gs == 0 || mbar_wait_abortable(pv_done, (gs - 1) & 1, status, abort_flag));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ws_ts(tbase, tQ + kk * 8, dK + kmajor_step(kk, kKB * kBoxBytes), idS, kk > 0 ? 1u : 0u);
          mma_commit(s_full);
          mma_commit(k_free);
          // P written, V landed, and before a row's first PV the previous row's O read
          ok = mbar_wait_abortable(p_full, gs & 1, status, abort_flag) &&
               mbar_wait_abortable(v_full, gs & 1, status, abort_flag) &&
               (j > 0 || lq == 0 || mbar_wait_abortable(o_free, (lq - 1) & 1, status, abort_flag));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ws_ts(tO, tbase + kk * 8, dV + uint64_t((kk * 2048) >> 4), idO, (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(pv_done);
        }
        ++lq;
      }
      // every product this thread issued has completed before TMEM is released
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, status);
    }
  } else {
    // ------------------------------------------------------------ softmax
    // The four warps run the same control flow whatever their waits return
    // (after a timeout the waits give up at once and the values are
    // discarded), so their named barriers always match.
    const int sp = warp & 3;  // TMEM lane quarter of this warp
    const int Ln = sp * 32 + lane;
    const int m = Ln & 63, kh = Ln >> 6;
    const uint32_t lane_off = uint32_t(sp * 32) << 16;
    const int tid = threadIdx.x - 64;
    // the next row of the stride with work from `r` on; empty rows on the way
    // get their outputs. (b0, b1): row_ptr[r], row_ptr[r + 1], read in advance
    auto seek = [&](int r, int b0, int b1, int& beg, int& cnt, int& nsteps) -> int {
      for (bool first = true; r < rows; r += gridDim.x, first = false) {
        if (first) {
          beg = b0;
          cnt = b1 - b0;
          if (cnt < 0 || cnt > g.n_blocks) {
            atomicOr(status, kDevErrBounds);
            cnt = 0;
          }
        } else {
          cnt = row_list(P, r, &beg);
        }
        nsteps = (cnt + kKB - 1) / kKB;
        if (nsteps == 0) {
          write_empty_row<D>(P, r % g.n_blocks, r / g.n_blocks, tid);
          continue;
        }
        if (small_takes(P, nsteps)) return r;
      }
      return rows;
    };
    // Q becomes the A operand of every S product of its row: both column halves of this lane's row
    auto q_to_tmem = [&](int lq) {
      mbar_wait_abortable(q_full, lq & 1, status, abort_flag);
      tile_to_tmem_a<D>(sm + L::kQ, tQ + lane_off, m, 0);
      tile_to_tmem_a<D>(sm + L::kQ, tQ + lane_off, m, 1);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qa_full);
    };
    int beg = 0, cnt = 0, nsteps = 0;
    int row = blockIdx.x < rows ? seek(blockIdx.x, __ldg(P.row_ptr + blockIdx.x), __ldg(P.row_ptr + blockIdx.x + 1),
                                       beg, cnt, nsteps)
                                : rows;
    if (row < rows) q_to_tmem(0);
    int lq = 0, gs = 0;
    while (row < rows) {
      const int I = row % g.n_blocks, head = row / g.n_blocks;
      const int sI = safe_shape(g, P.zone_shape, I, status);  // read now, used in the epilogue
      // the list bounds of the next row of the stride, read now, used after the steps
      const int pr = row + gridDim.x;
      const int pb0 = pr < rows ? __ldg(P.row_ptr + pr) : 0, pb1 = pr < rows ? __ldg(P.row_ptr + pr + 1) : 0;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < nsteps; ++j, ++gs) {
        const bool valid = (j * kKB + kh) < cnt;  // warp-uniform: kh is fixed per warp
        uint64_t members = ~uint64_t(0);
        if (g.partial && valid) members = key_block_members(g, P.zone_shape, __ldg(P.col_idx + beg + j * kKB + kh));
        mbar_wait_abortable(s_full, gs & 1, status, abort_flag);
        tc_fence_after();
        uint32_t r[64];
        tmem_ld32(tbase + lane_off, r);
        tmem_ld32(tbase + lane_off + 32, r + 32);
        tmem_ld_wait();
        mask_scores32(r, uint32_t(members));
        mask_scores32(r + 32, uint32_t(members >> 32));
        const float mx = valid ? max64(r) * P.scale_log2 : -INFINITY;
        const float m_new = fmaxf(m_run, mx);
        const bool resc = m_new > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, resc)) {
          const float alpha = resc ? fast_exp2(m_run - m_new) : 1.f;
          if (resc) {
            l_run *= alpha;
            m_run = m_new;
          }
          if (j > 0) {
            // O holds the row's PV of the previous step, complete: this S was issued after it
#pragma unroll
            for (int h = 0; h < D / 32; ++h) {
              uint32_t o[32];
              const uint32_t ta = tO + lane_off + h * 32;
              tmem_ld32(ta, o);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st16(ta, o);
              tmem_st16(ta + 16, o + 16);
            }
            tmem_st_wait();
          }
        }
        uint32_t pk[32];
        if (valid) {
          const float c = P.scale_log2, nm = m_run == -INFINITY ? 0.f : -m_run;
          float la = 0.f, lb = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(r[2 * i]), c, nm));
            const float p1 = fast_exp2(fmaf(__uint_as_float(r[2 * i + 1]), c, nm));
            la += p0;
            lb += p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          l_run += la + lb;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) pk[i] = 0u;
        }
        // P over the first 32 columns of S (every S value of this lane was read above)
        tmem_st16(tbase + lane_off, pk);
        tmem_st16(tbase + lane_off + 16, pk + 16);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      // every S product of this row has completed: the next row's Q may take the Q columns
      int nbeg = 0, ncnt = 0, nns = 0;
      const int nrow = seek(pr, pb0, pb1, nbeg, ncnt, nns);
      if (nrow < rows) q_to_tmem(lq + 1);
      // ---------------------------------------------------------- epilogue
      mbar_wait_abortable(pv_done, (gs - 1) & 1, status, abort_flag);
      tc_fence_after();
      redm[kh * 64 + m] = m_run;
      redl[kh * 64 + m] = l_run;
      // the previous row's output tile has left the exchange buffer
      if (P.tma_out && tid == 0) bulk_wait_group_read0();
      named_bar_sync(1, 128);
      const bool ok = *abort_flag == 0;
      const float M = fmaxf(redm[m], redm[64 + m]);
      float Lsum = 0.f;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float lq2 = redl[q * 64 + m];
        if (lq2 > 0.f) Lsum += lq2 * fast_exp2(redm[q * 64 + m] - M);
      }
      const float inv = (Lsum > 0.f && ok) ? 1.f / Lsum : 0.f;
      const float w = l_run > 0.f ? fast_exp2(m_run - M) * inv : 0.f;  // weight of this lane's part
      // this thread keeps channel half kh of row m and hands half kh ^ 1 to the
      // other lane half, kXC channels per round
      constexpr int NC = D / 2;
      float ov[NC];
#pragma unroll
      for (int c0 = 0; c0 < NC; c0 += L::kXC) {
        float gv[L::kXC];
        tmem_ld_f<L::kXC>(tO + lane_off + (kh ^ 1) * NC + c0, gv);
        tmem_ld_f<L::kXC>(tO + lane_off + kh * NC + c0, ov + c0);
        if (c0 + L::kXC == NC) {
          // this warp's last read of O: the next row's first PV may overwrite it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_free);
        }
        float* xo = X + ((kh ^ 1) * 64 + m) * L::kXPitch;
#pragma unroll
        for (int i = 0; i < L::kXC / 4; ++i)
          reinterpret_cast<float4*>(xo)[i] =
              make_float4(gv[4 * i] * w, gv[4 * i + 1] * w, gv[4 * i + 2] * w, gv[4 * i + 3] * w);
        named_bar_sync(1, 128);
        const float* xi = X + (kh * 64 + m) * L::kXPitch;
#pragma unroll
        for (int i = 0; i < L::kXC / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(xi)[i];
          ov[c0 + 4 * i] = fmaf(ov[c0 + 4 * i], w, t.x);
          ov[c0 + 4 * i + 1] = fmaf(ov[c0 + 4 * i + 1], w, t.y);
          ov[c0 + 4 * i + 2] = fmaf(ov[c0 + 4 * i + 2], w, t.z);
          ov[c0 + 4 * i + 3] = fmaf(ov[c0 + 4 * i + 3], w, t.w);
        }
        named_bar_sync(1, 128);  // the exchange buffer is free for the next round (and row)
      }
#pragma unroll
      for (int i = 0; i < NC; ++i) ov[i] = inv == 0.f ? 0.f : ov[i];
      const BlockBox qb = block_box(g, sI, I);
      const int tok = block_token(g, qb, m);
      const bool row_in = !g.partial || block_slot_in_grid(g, qb, m);
      if (P.tma_out) {
        // bf16 rows of the block into swizzled [dh][64][128 B] tiles, O over
        // the exchange buffer and its rounding residual over the Q tile (free:
        // the next row's Q is in TMEM, and the copy warp stages the row after
        // it only once these box stores have read the tile), then one box
        // store per 64 channels and tile (rows outside the grid fall outside
        // the tensor and are not written)
        const int dh = (kh * NC) / 64, c0 = ((kh * NC) % 64) / 8;
#pragma unroll
        for (int q = 0; q < NC / 8; ++q) {
          const uint32_t so = dh * kBoxBytes + sw128_offset(m, c0 + q);
          const float* x = ov + 8 * q;
          *reinterpret_cast<uint4*>(sm + L::kX + so) =
              make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                         pack_bf16x2(x[6], x[7]));
          if (stage_lo) {
            float t[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) t[i] = x[i] - __bfloat162float(__float2bfloat16_rn(x[i]));
            *reinterpret_cast<uint4*>(sm + L::kQ + so) =
                make_uint4(pack_bf16x2(t[0], t[1]), pack_bf16x2(t[2], t[3]), pack_bf16x2(t[4], t[5]),
                           pack_bf16x2(t[6], t[7]));
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (tid == 0) {
          for (int h = 0; h < D / 64; ++h) {
            tma_store_5d(&P.mo[sI], sm + L::kX + h * kBoxBytes, h * 64, head, qb.w0, qb.h0, qb.t0);
            if (stage_lo) tma_store_5d(&P.mol[sI], sm + L::kQ + h * kBoxBytes, h * 64, head, qb.w0, qb.h0, qb.t0);
          }
          bulk_commit_group();
          if (stage_lo) {
            bulk_wait_group_read0();
            mbar_arrive(stage_free);
          }
        }
      } else if (row_in) {
        const int64_t off = int64_t(tok) * P.tok_stride + int64_t(head) * D + kh * NC;
        store_row<NC>(P.o, off, ov, P.out_fp32);
        if (P.o_lo) {
          float lo[NC];
#pragma unroll
          for (int i = 0; i < NC; ++i) lo[i] = ov[i] - __bfloat162float(__float2bfloat16_rn(ov[i]));
          store_row<NC>(P.o_lo, off, lo, false);
        }
      }
      if (row_in) {
        if (kh == 0) {
          const int N = g.T * g.H * g.W;
          P.lse[int64_t(head) * N + tok] = (Lsum > 0.f && ok) ? (M + log2f(Lsum)) * 0.69314718055994531f : -INFINITY;
        }
      }
      ++lq;
      row = nrow;
      beg = nbeg;
      cnt = ncnt;
      nsteps = nns;
    }
    // the last output tile has been read before the CTA's shared memory goes
    if (P.tma_out && tid == 0) bulk_wait_group_read0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, L::kTmemCols);
  }
}

// fp32 -> bf16 staging copy of a token-major tensor (contiguous output).
__global__ void to_bf16_kernel(const float* __restrict__ src, int64_t tok_stride, int C, int64_t n_tokens,
                               __nv_bfloat16* __restrict__ dst) {
  const int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i >= n_tokens * C) return;
  const int64_t n = i / C, c = i - n * C;
  const float4 v = *reinterpret_cast<const float4*>(src + n * tok_stride + c);
  uint2 out = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  *reinterpret_cast<uint2*>(dst + i) = out;
}

// Block-major operand images (layout in host.h): one CTA per (block, head),
// 128 threads, D/16 independent 16-byte loads per thread; sixteen consecutive
// threads (D = 128) read one token's 256-byte head slice.
template <int D>
__global__ void __launch_bounds__(128) block_images_kernel(const Geo g, const int32_t* __restrict__ zone_shape,
                                                           const __nv_bfloat16* __restrict__ src, int64_t tok_stride,
                                                           uint8_t* __restrict__ dst, int* status) {
  constexpr int CPR = D / 8;            // 16-byte chunks per row
  constexpr int PER = 64 * CPR / 128;   // chunks per thread
  const int b = blockIdx.x, head = blockIdx.y;
  const int s = safe_shape(g, zone_shape, b, status);
  const BlockBox bb = block_box(g, s, b);
  uint8_t* img = dst + image_offset(g, head, b, D);
  uint4 v[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + 128 * k;
    const int r = i / CPR, c = i % CPR;
    v[k] = make_uint4(0u, 0u, 0u, 0u);
    if (!g.partial || block_slot_in_grid(g, bb, r)) {
      const int tok = block_token(g, bb, r);
      v[k] = __ldg(reinterpret_cast<const uint4*>(src + int64_t(tok) * tok_stride + int64_t(head) * D + c * 8));
    }
  }
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int i = threadIdx.x + 128 * k;
    const int r = i / CPR, c = i % CPR;
    *reinterpret_cast<uint4*>(img + (c / 8) * kBoxBytes + sw128_offset(r, c % 8)) = v[k];
  }
}

}  // namespace

size_t block_images_bytes(const Geo& g, int heads, int head_dim) {
  return size_t(heads) * g.n_blocks * size_t(head_dim) * 128u;
}

prism_status launch_block_images(const Geo& g, const int32_t* zone_shape, const void* src, int64_t tok_stride,
                                 int heads, int head_dim, void* dst, int* status, cudaStream_t s) {
  const dim3 grid(g.n_blocks, heads);
  const auto* sp = static_cast<const __nv_bfloat16*>(src);
  auto* dp = static_cast<uint8_t*>(dst);
  if (head_dim == 128)
    block_images_kernel<128><<<grid, 128, 0, s>>>(g, zone_shape, sp, tok_stride, dp, status);
  else if (head_dim == 64)
    block_images_kernel<64><<<grid, 128, 0, s>>>(g, zone_shape, sp, tok_stride, dp, status);
  else
    return PRISM_ERR_UNSUPPORTED;
  return cuda_status(cudaGetLastError());
}

prism_status stage_bf16(const void* src, prism_dtype dtype, int64_t tok_stride, int C, int64_t n_tokens,
                        __nv_bfloat16* dst, cudaStream_t s) {
  if (dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
  const int64_t total = n_tokens * C / 4;
  to_bf16_kernel<<<unsigned((total + 255) / 256), 256, 0, s>>>(static_cast<const float*>(src), tok_stride, C, n_tokens,
                                                               dst);
  return cuda_status(cudaGetLastError());
}

// Workspace: [fp32 input only: bf16 copies of q, k, v] + block images of k and v.
size_t bsa_fwd_ws_bytes(const Geo& g, int heads, int head_dim, prism_dtype dtype) {
  WsCarver c;
  if (dtype == PRISM_FP32) {
    const size_t t = size_t(g.T) * g.H * g.W * heads * head_dim * 2;
    c.take(t); c.take(t); c.take(t);
  }
  c.take(block_images_bytes(g, heads, head_dim));
  c.take(block_images_bytes(g, heads, head_dim));
  return c.off;
}

}  // namespace prism

using namespace prism;

extern "C" prism_status prism_bsa_fwd(const prism_geometry* geo, const int32_t* zone_shape, const void* q,
                                      const void* k, const void* v, prism_dtype dtype, int32_t heads,
                                      int32_t head_dim, int64_t tok_stride, float scale, const int32_t* row_ptr,
                                      const int32_t* col_idx, int64_t nnz, void* o, float* lse, void* o_lo,
                                      void* ws, size_t ws_bytes, void* stream) {
  Geo g;
  prism_status st = make_geo(geo, &g);
  if (st != PRISM_OK) return st;
  if (!zone_shape || !q || !k || !v || !row_ptr || !col_idx || !o || !lse) return PRISM_ERR_ARG;
  if (dtype != PRISM_BF16 && dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
  if (head_dim != 64 && head_dim != 128) return PRISM_ERR_UNSUPPORTED;
  if (heads < 1 || heads > 65535) return PRISM_ERR_UNSUPPORTED;
  if (tok_stride < int64_t(heads) * head_dim || tok_stride % 8) return PRISM_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return PRISM_ERR_ARG;
  if (nnz < -1) return PRISM_ERR_ARG;
  for (const void* p : {q, k, v, static_cast<const void*>(o), static_cast<const void*>(o_lo)})
    if (reinterpret_cast<uintptr_t>(p) % 16) return PRISM_ERR_ARG;
  const size_t need = bsa_fwd_ws_bytes(g, heads, head_dim, dtype);
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < need) return PRISM_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const void* qb = q;
  const void* kb = k;
  const void* vb = v;
  int64_t in_stride = tok_stride;
  WsCarver c;
  if (dtype == PRISM_FP32) {
    const int64_t N = int64_t(g.T) * g.H * g.W;
    const int C = heads * head_dim;
    const size_t t = size_t(N) * C * 2;
    __nv_bfloat16* sq = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + c.take(t));
    __nv_bfloat16* sk = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + c.take(t));
    __nv_bfloat16* sv = reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + c.take(t));
    if ((st = stage_bf16(q, dtype, tok_stride, C, N, sq, s)) != PRISM_OK) return st;
    if ((st = stage_bf16(k, dtype, tok_stride, C, N, sk, s)) != PRISM_OK) return st;
    if ((st = stage_bf16(v, dtype, tok_stride, C, N, sv, s)) != PRISM_OK) return st;
    qb = sq; kb = sk; vb = sv;
    in_stride = C;
  }
  // The plan. Sparse (a known nnz of at most kSparseBlocksPerRow key blocks
  // per row on average): the short-row kernel takes every row and gathers K
  // and V through 5-D tensor maps; each key block is read by few rows, so
  // making block images would cost more than it saves. Otherwise K and V are
  // made block images first: every key block the kernels gather is then one
  // contiguous bulk copy per 64 channels instead of 64 scattered token rows;
  // the short rows go to the short-row kernel and the long ones to
  // bsa_fwd_kernel. Both plans compute the same result.
  const int64_t rows = int64_t(heads) * g.n_blocks;
  const bool all_rows = nnz >= 0 && nnz <= kSparseBlocksPerRow * rows;
  uint8_t* kimg = static_cast<uint8_t*>(ws) + c.take(block_images_bytes(g, heads, head_dim));
  uint8_t* vimg = static_cast<uint8_t*>(ws) + c.take(block_images_bytes(g, heads, head_dim));
  if (!all_rows) {
    if ((st = launch_block_images(g, zone_shape, kb, in_stride, heads, head_dim, kimg, ws_status(ws), s)) != PRISM_OK)
      return st;
    if ((st = launch_block_images(g, zone_shape, vb, in_stride, heads, head_dim, vimg, ws_status(ws), s)) != PRISM_OK)
      return st;
  }
  FwdParams P;
  std::memset(&P, 0, sizeof(P));
  const bool tma_out = dtype == PRISM_BF16;
  for (int ci = 0; ci < g.n_cand; ++ci) {
    const int bt = g.cand[ci][0], bh = g.cand[ci][1], bw = g.cand[ci][2];
    if ((st = encode_block_map(&P.mq[ci], qb, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
    if (all_rows) {
      if ((st = encode_block_map(&P.mk[ci], kb, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
      if ((st = encode_block_map(&P.mv[ci], vb, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
    }
    if (tma_out) {
      if ((st = encode_block_map(&P.mo[ci], o, g, heads, head_dim, tok_stride, bt, bh, bw)) != PRISM_OK) return st;
      if (o_lo && (st = encode_block_map(&P.mol[ci], o_lo, g, heads, head_dim, tok_stride, bt, bh, bw)) != PRISM_OK)
        return st;
    }
  }
  P.tma_out = tma_out ? 1 : 0;
  P.kimg = kimg;
  P.vimg = vimg;
  P.g = g;
  P.zone_shape = zone_shape;
  P.row_ptr = row_ptr;
  P.col_idx = col_idx;
  P.o = o;
  P.lse = lse;
  P.o_lo = dtype == PRISM_BF16 ? static_cast<__nv_bfloat16*>(o_lo) : nullptr;
  P.status = ws_status(ws);
  P.tok_stride = tok_stride;
  P.scale_log2 = scale * 1.4426950408889634f;
  P.out_fp32 = dtype == PRISM_FP32;
  P.heads = heads;
  P.all_rows = all_rows ? 1 : 0;
  // long rows: one CTA per row, launched in row order (neighbouring rows share key blocks in L2);
  // short and empty rows (every row in the sparse plan): two CTAs per SM, each looping over its rows
  const dim3 grid(g.n_blocks, heads);
  const dim3 grid_small(unsigned(std::min<int64_t>(rows, 2 * device_sm_count())));
  // short and empty rows first (two CTAs per SM), then, in the dense plan, the long rows
  if (head_dim == 128) {
    const size_t smem = FwdSmallSmem<128>::kTotal + 1024;
    if (cudaFuncSetAttribute(bsa_fwd_small_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
      return PRISM_ERR_CUDA;
    bsa_fwd_small_kernel<128><<<grid_small, kSmallThreads, smem, s>>>(P);
  } else {
    const size_t smem = FwdSmallSmem<64>::kTotal + 1024;
    if (cudaFuncSetAttribute(bsa_fwd_small_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
      return PRISM_ERR_CUDA;
    bsa_fwd_small_kernel<64><<<grid_small, kSmallThreads, smem, s>>>(P);
  }
  if (all_rows) return cuda_status(cudaGetLastError());
  if (head_dim == 128) {
    const size_t smem = FwdSmem<128>::kTotal + 1024;
    if (cudaFuncSetAttribute(bsa_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
      return PRISM_ERR_CUDA;
    bsa_fwd_kernel<128><<<grid, kFwdThreads, smem, s>>>(P);
  } else {
    const size_t smem = FwdSmem<64>::kTotal + 1024;
    if (cudaFuncSetAttribute(bsa_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
        cudaSuccess)
      return PRISM_ERR_CUDA;
    bsa_fwd_kernel<64><<<grid, kFwdThreads, smem, s>>>(P);
  }
  return cuda_status(cudaGetLastError());
}
