// a7: block-sparse attention backward with the block selection held fixed.
//
// Prism is a training method (README "Overview": natively training joint
// video-audio models with the sparse attention), so the attention over the
// selected blocks needs dQ, dK and dV. With P_ij = exp(scale q_i.k_j - lse_i)
// on the selected blocks and D_i = rowsum(dO_i * O_i):
//   dV_j = sum_i P_ij dO_i,  dS_ij = P_ij (dO_i . v_j - D_i),
//   dQ_i = scale sum_j dS_ij k_j,  dK_j = scale sum_i dS_ij q_i.
//
// Kernels:
//   prep        one CTA per (block, head): D in block order and the forward
//               LSE converted to log2 units in block order;
//   csc_scatter the CSR selection transposed into a bitmask [head, J, I];
//               csc_count + scan + list fill give the CSC (ascending I);
//   dq          one CTA per (query block, head), q-stationary: per step of two
//               selected key blocks, S = Q K^T and dP = dO V^T (.ws M=64,
//               N=128), then dS in the softmax warps (written back into
//               TMEM), then dQ += dS K (.ws M=64, dS as the TMEM A operand);
//               dQ lives in TMEM for the whole row;
//   dkdv        one CTA per (key block, head), kv-stationary over the query
//               blocks that selected it: S^T = K Q^T, dP^T = V dO^T, then
//               P^T, dS^T in the softmax warps (written back into TMEM), then
//               dV += P^T dO and dK += dS^T Q (.ws M=64, P^T / dS^T as TMEM A
//               operands); dK, dV live in TMEM.
// Both passes issue their products from two threads and run the softmax in
// two warp groups on alternate steps. Splitting dQ from dK/dV costs one
// recomputation of S and dP but needs no atomics and is deterministic. Each
// pass streams its two operands (K and V, or Q and dO) as bulk copies of
// block images made just before it; the tiles a CTA keeps for its whole life
// (Q / dO in dq, K / V in dkdv) come through 5-D tensor maps.
#include <cuda_bf16.h>

#include <cmath>
#include <cstring>
#include <type_traits>

#include "bsa_common.cuh"
#include "host.h"

namespace prism {
namespace {

constexpr int kKB = 2;
constexpr int kSoftWarps = 8;
constexpr int kGroupWarps = 4;  // the softmax warps form two groups taking alternate steps
constexpr int kBwdThreads = 64 + 32 * kSoftWarps + 32;
constexpr int kIssuerB = 2 + kSoftWarps;  // warp of the second MMA issuer

struct BwdParams {
  CUtensorMap mq[kMaxCand];
  CUtensorMap mk[kMaxCand];
  CUtensorMap mv[kMaxCand];
  CUtensorMap mdo[kMaxCand];
  // bf16 outputs in the sparse plan: dq (dq pass) or dk and dv (dkdv pass), stored as 5-D boxes
  CUtensorMap mo0[kMaxCand];
  CUtensorMap mo1[kMaxCand];
  // block images (layout in host.h) of the two operands a kernel streams:
  // K and V for dq, Q and dO for dkdv
  const uint8_t* img0;
  const uint8_t* img1;
  Geo g;
  const int32_t* zone_shape;
  const int32_t* ptr;  // CSR row_ptr (dq) or CSC col_ptr (dkdv), over (head, block)
  const int32_t* idx;  // CSR col_idx (dq) or CSC row_idx (dkdv)
  const float* lse2;   // [heads, n_blocks, 64] LSE * log2(e), block order
  const float* dvec;   // [heads, n_blocks, 64] rowsum(dO * O), block order
  void* out0;          // dq   | dk
  void* out1;          //      | dv
  int* status;
  int64_t tok_stride;  // of the outputs, elements
  float scale_log2;
  float scale;
  int out_fp32;
  int heads;
};

// List of row (or column) `row` of ptr / idx: its first entry and its length
// (a malformed length is reported and read as 0).
__device__ __forceinline__ int bwd_list(const BwdParams& P, int row, int* beg) {
  const int b = __ldg(P.ptr + row);
  int cnt = __ldg(P.ptr + row + 1) - b;
  if (cnt < 0 || cnt > P.g.n_blocks) {
    atomicOr(P.status, kDevErrBounds);
    cnt = 0;
  }
  *beg = b;
  return cnt;
}

// The rows of an output block leave as box stores for bf16 outputs: each
// thread writes its NC channels (from `c`) of row m, rounded to bf16, into a
// swizzled [D/64][64][128 B] tile; once every thread has written, one thread
// stores the tile with one box per 64 channels (slots outside the grid fall
// outside the tensor and are not written).
template <int NC>
__device__ __forceinline__ void tile_put_row(uint8_t* tile, int m, int c, const float* v) {
  const int dh = c / 64, c0 = (c % 64) / 8;
#pragma unroll
  for (int q = 0; q < NC / 8; ++q) {
    const float* x = v + 8 * q;
    *reinterpret_cast<uint4*>(tile + dh * kBoxBytes + sw128_offset(m, c0 + q)) =
        make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                   pack_bf16x2(x[6], x[7]));
  }
}

// One step slot of the two streamed operands (Q and dO for dkdv) of block b,
// each laid out [dh][block][64][128 B] from dst0 / dst1: bulk copies of the
// block images, or (G, the sparse plan) 5-D tensor-map copies from the box
// origin {shape, t0, h0, w0} cached with the block id. The plan is a template
// parameter: a run-time test in the copy loop cost the dense plan's dK/dV and
// dQ passes about 2 % at 2K.
template <int D, bool G>
__device__ __forceinline__ void stream_pair(const BwdParams& P, const CUtensorMap* map0, const CUtensorMap* map1,
                                            uint8_t* dst0, uint8_t* dst1, int slot, int head, int b, int4 box,
                                            uint64_t* bar) {
  if constexpr (G) {
    for (int dh = 0; dh < D / 64; ++dh) {
      const uint32_t off = dh * (kKB * kBoxBytes) + slot * kBoxBytes;
      tma_load_5d(dst0 + off, &map0[box.x], bar, dh * 64, head, box.w, box.z, box.y);
      tma_load_5d(dst1 + off, &map1[box.x], bar, dh * 64, head, box.w, box.z, box.y);
    }
  } else {
    const size_t io = image_offset(P.g, head, b, D);
    for (int dh = 0; dh < D / 64; ++dh) {
      const uint32_t off = dh * (kKB * kBoxBytes) + slot * kBoxBytes;
      bulk_load(dst0 + off, P.img0 + io + dh * kBoxBytes, kBoxBytes, bar);
      bulk_load(dst1 + off, P.img1 + io + dh * kBoxBytes, kBoxBytes, bar);
    }
  }
}

// ----------------------------------------------------------------------- dq
// Three slots, each holding K and V of one step (two key blocks) from its load
// until the dQ product of that step completes. Q and dO are staged through
// shared memory once and copied into TMEM (the A operands of every S / dP
// product).
// The softmax warps form two groups of four taking alternate steps (group
// j % 2 takes step j), one thread per TMEM lane: the thread in lane m + 64 kh
// holds row m of S_j and dP_j against key block kh of the step (64 values
// each) and writes dS (bf16) back over the first 32 columns of its group's S
// buffer. dS is thus the TMEM A operand of the dQ product, and the .ws lane
// split makes lane half kh accumulate the key-block-kh part of dQ: the B
// operand's two 64-column halves are the same 64 channels of K of key block 0
// and of key block 1. The two parts are added once, in the epilogue.
// Two threads issue the products, each in step order: warp 1 issues
// A_j = (S_j = Q K_j^T, dP_j = dO V_j^T) into group (j % 2)'s buffers once
// slot j has landed and that group's previous dQ product (which read dS from
// the same buffer) has completed; warp 10 issues B_j = (dQ_parts += dS_j K_j)
// once dS_j is written. While one waits on a barrier the other's products keep
// the tensor pipe busy.
template <int D>
struct DqSmem {
  static constexpr uint32_t kQD = 0;               // Q, dO staging [2][dh][64][128 B]
  static constexpr uint32_t kQDBytes = 2 * D * 128;
  static constexpr uint32_t kHalf = kKB * D * 128;   // K (or V) of one step, [dh][key block][64][128 B]
  static constexpr uint32_t kSlotBytes = 2 * kHalf;  // K then V
  static constexpr int kSlots = 3;
  static constexpr uint32_t kSlot0 = kQDBytes;
  static constexpr uint32_t kDesc = kSlot0 + kSlots * kSlotBytes;  // block-id ring
  static constexpr uint32_t kBar = kDesc + kDescRing * 4;
  static constexpr uint32_t kTotal = kBar + 256;
  // epilogue exchange of dQ part quarters: [kh][group][64 rows][D/4 + 4 floats], over the slots,
  // then the bf16 dQ tile
  static constexpr uint32_t kXPitch = D / 4 + 4;
  static constexpr uint32_t kXTile = (4 * 64 * kXPitch * 4 + 1023) / 1024 * 1024;
  static_assert(kXTile + D * 128 <= kSlots * kSlotBytes, "exchange buffer and tile fit the slots");
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) bsa_dq_kernel(const __grid_constant__ BwdParams P) {
  using L = DqSmem<D>;
  constexpr int NS = L::kSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* qd_full = bars + 0;
  uint64_t* kv_full = bars + 1;    // [3] K and V of the slot's step landed
  uint64_t* kv_free = bars + 4;    // [3] dQ product of the slot's step complete
  uint64_t* s_full = bars + 7;     // [2] per group: its A complete
  uint64_t* ds_full = bars + 9;    // [2] per group: its dS written to TMEM (4 warps)
  uint64_t* ds_free = bars + 11;   // [2] per group: its B complete (its S / dP buffers free)
  uint64_t* mma_done = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 15);
  uint64_t* qa_full = bars + 16;  // Q and dO copied into TMEM by the softmax warps
  uint64_t* b_done = bars + 17;   // every B product complete

  const Geo& g = P.g;
  const int I = blockIdx.x, head = blockIdx.y;
  const int row = head * g.n_blocks + I;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = P.status;
  const int beg = P.ptr[row];
  int cnt = P.ptr[row + 1] - beg;
  if (cnt < 0 || cnt > g.n_blocks) {
    if (threadIdx.x == 0) atomicOr(status, kDevErrBounds);
    cnt = 0;
  }
  const int nsteps = (cnt + kKB - 1) / kKB;
  if (threadIdx.x == 0) {
    mbar_init(qd_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&ds_full[i], kGroupWarps);
      mbar_init(&ds_free[i], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(b_done, 1);
    mbar_init(qa_full, kSoftWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // TMEM columns: S [2 groups x 64] at 0 (dS over its first 32), dP [2 x 64]
  // at 128, dQ parts at 256 (D columns), Q at 384, dO at 448
  const uint32_t tdQ = tbase + 256, tQ = tbase + 384, tDO = tbase + 448;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (nsteps > 0) {
      IdCache dc{reinterpret_cast<int*>(sm + L::kDesc), 0};
      if (lane == 0) {
        const int sI = safe_shape(g, P.zone_shape, I, status);
        const BlockBox qb = block_box(g, sI, I);
        mbar_arrive_expect_tx(qd_full, 2 * D * 128);
        for (int dh = 0; dh < D / 64; ++dh) {
          tma_load_5d(sm + L::kQD + dh * kBoxBytes, &P.mq[sI], qd_full, dh * 64, head, qb.w0, qb.h0, qb.t0);
          tma_load_5d(sm + L::kQD + D * 128 + dh * kBoxBytes, &P.mdo[sI], qd_full, dh * 64, head, qb.w0, qb.h0,
                      qb.t0);
        }
      }
      bool ok = true;
      int issued = 0;
      for (int j = 0; j < nsteps && ok; ++j) {
        dc.ensure(kKB * j + kKB - 1, g, P.idx, beg, cnt, status, lane);
        if (lane == 0) {
          const int s = j % NS;
          // slot s last held step j - 3: free once its dQ product completed
          if (j >= NS) ok = mbar_wait_abortable(&kv_free[s], ((j / NS) - 1) & 1, status, abort_flag);
          if (ok) {
            uint8_t* dst = sm + L::kSlot0 + s * L::kSlotBytes;
            mbar_arrive_expect_tx(&kv_full[s], L::kSlotBytes);
            for (int slot = 0; slot < kKB; ++slot) {
              const size_t io = image_offset(g, head, dc.get(kKB * j + slot), D);
              for (int dh = 0; dh < D / 64; ++dh) {
                const uint32_t off = dh * (kKB * kBoxBytes) + slot * kBoxBytes;
                bulk_load(dst + off, P.img0 + io + dh * kBoxBytes, kBoxBytes, &kv_full[s]);
                bulk_load(dst + L::kHalf + off, P.img1 + io + dh * kBoxBytes, kBoxBytes, &kv_full[s]);
              }
            }
            issued = j + 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      if (lane == 0) {
        // drain: every issued copy has landed before the CTA may exit
        mbar_wait(qd_full, 0, status);
        for (int i = issued - NS > 0 ? issued - NS : 0; i < issued; ++i)
          mbar_wait(&kv_full[i % NS], (i / NS) & 1, status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ A issuer
    if (lane == 0 && nsteps > 0) {
      const uint32_t idS = idesc_bf16_f32(64, 64 * kKB, false, false);
      const uint32_t sK0 = smem_u32(sm + L::kSlot0);
      const uint64_t dK0 = sdesc_sw128(sK0, 16, 1024);             // K as B of S
      const uint64_t dV0 = sdesc_sw128(sK0 + L::kHalf, 16, 1024);  // V as B of dP
      constexpr uint64_t kSlotStep = L::kSlotBytes >> 4;
      bool ok = mbar_wait_abortable(qa_full, 0, status, abort_flag);
      // A_j: S_j and dP_j into group (j % 2)'s buffers, once slot j has landed
      // and that group's previous B (which read dS from the S buffer) completed
      for (int j = 0; j < nsteps && ok; ++j) {
        ok = mbar_wait_abortable(&kv_full[j % NS], (j / NS) & 1, status, abort_flag) &&
             mbar_wait_abortable(&ds_free[j & 1], ((j >> 1) & 1) ^ 1, status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t so = uint64_t(j % NS) * kSlotStep;
        const uint32_t tS = tbase + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ws_ts(tS, tQ + kk * 8, dK0 + so + kmajor_step(kk, kKB * kBoxBytes), idS, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ws_ts(tS + 128, tDO + kk * 8, dV0 + so + kmajor_step(kk, kKB * kBoxBytes), idS, kk > 0 ? 1u : 0u);
        mma_commit(&s_full[j & 1]);
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, status);
    }
  } else if (warp == kIssuerB) {
    // ------------------------------------------------------------ B issuer
    if (lane == 0 && nsteps > 0) {
      // B = K of the step, MN-major, N = 128: 64 channels of key block 0
      // then the same channels of key block 1 (LBO = the block stride)
      const uint32_t idQ = idesc_bf16_f32(64, 128, false, true);
      const uint64_t dKmn0 = sdesc_sw128(smem_u32(sm + L::kSlot0), kBoxBytes, 1024);
      constexpr uint64_t kSlotStep = L::kSlotBytes >> 4;
      bool ok = true;
      // B_j once dS_j is written (which implies A_j, hence slot j, complete)
      for (int j = 0; j < nsteps && ok; ++j) {
        ok = mbar_wait_abortable(&ds_full[j & 1], (j >> 1) & 1, status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t so = uint64_t(j % NS) * kSlotStep;
        const uint32_t tDS = tbase + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            mma_ws_ts(tdQ + c * 64, tDS + kk * 8, dKmn0 + so + uint64_t((c * kKB * kBoxBytes + kk * 2048) >> 4), idQ,
                      (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&kv_free[j % NS]);
        mma_commit(&ds_free[j & 1]);
      }
      mma_commit(b_done);
      mbar_wait(b_done, 0, status);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 2, grp = sw / kGroupWarps, sp = warp & 3;
    const int Ln = sp * 32 + lane;
    const int m = Ln & 63, kh = Ln >> 6;
    const uint32_t lane_off = uint32_t(sp * 32) << 16;
    const float lse2 = P.lse2[size_t(row) * 64 + m];
    const float dm = P.dvec[size_t(row) * 64 + m];
    if (nsteps > 0) {
      // Q and dO are the A operands of every S / dP product: one copy into
      // TMEM (the two groups copy the two column halves)
      mbar_wait_abortable(qd_full, 0, status, abort_flag);
      tile_to_tmem_a<D>(sm + L::kQD, tQ + lane_off, m, grp);
      tile_to_tmem_a<D>(sm + L::kQD + D * 128, tDO + lane_off, m, grp);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qa_full);
    }
    int k = 0;  // this group's step count
    for (int j = grp; j < nsteps; j += 2, ++k) {
      const bool valid = (j * kKB + kh) < cnt;  // warp-uniform
      // keys of a key block clipped by the grid's edge (read before the wait)
      uint64_t members = ~uint64_t(0);
      if (g.partial && valid) members = key_block_members(g, P.zone_shape, __ldg(P.idx + beg + j * kKB + kh));
      mbar_wait_abortable(&s_full[grp], k & 1, status, abort_flag);
      tc_fence_after();
      uint32_t pk[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t rs[32], rp[32];
        tmem_ld32(tbase + lane_off + grp * 64 + h * 32, rs);
        tmem_ld32(tbase + lane_off + 128 + grp * 64 + h * 32, rp);
        tmem_ld_wait();
        mask_scores32(rs, uint32_t(members >> (32 * h)));  // P = exp2(-inf) = 0 there, hence dS = 0
        if (valid) {
          const float c = P.scale_log2, nl = -lse2;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(rs[2 * i]), c, nl));
            const float p1 = fast_exp2(fmaf(__uint_as_float(rs[2 * i + 1]), c, nl));
            pk[16 * h + i] =
                pack_bf16x2(p0 * (__uint_as_float(rp[2 * i]) - dm), p1 * (__uint_as_float(rp[2 * i + 1]) - dm));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[16 * h + i] = 0u;
        }
      }
      // dS over the first 32 columns of the S buffer (every S / dP value of
      // this lane was read above)
      tmem_st16(tbase + lane_off + grp * 64, pk);
      tmem_st16(tbase + lane_off + grp * 64 + 16, pk + 16);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full[grp]);
    }
    // ---------------------------------------------------------- epilogue
    // this group's last B complete; once both groups are here every product
    // is complete and the slots hold the exchange buffer
    if (k > 0) mbar_wait_abortable(&ds_free[grp], (k - 1) & 1, status, abort_flag);
    tc_fence_after();
    named_bar_sync(1, 32 * kSoftWarps);
    const bool ok = *abort_flag == 0;
    // This thread holds the key-block-kh part of dQ row m; it keeps channel
    // quarter grp * 2 + kh and hands quarter grp * 2 + (kh ^ 1) to the thread
    // of the other lane half.
    constexpr int NC = D / 4;
    const int keep = grp * (D / 2) + kh * NC, give = grp * (D / 2) + (kh ^ 1) * NC;
    float v[NC];
    if (nsteps > 0) {  // uniform; on an abort the values are discarded below
      float gv[NC];
      tmem_ld_f<NC>(tdQ + lane_off + give, gv);
      tmem_ld_f<NC>(tdQ + lane_off + keep, v);
      float* xo = reinterpret_cast<float*>(sm + L::kSlot0) + ((kh * 2 + grp) * 64 + m) * L::kXPitch;
#pragma unroll
      for (int i = 0; i < NC / 4; ++i)
        reinterpret_cast<float4*>(xo)[i] = make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]);
      named_bar_sync(1, 32 * kSoftWarps);
      const float* xi = reinterpret_cast<const float*>(sm + L::kSlot0) + (((kh ^ 1) * 2 + grp) * 64 + m) * L::kXPitch;
#pragma unroll
      for (int i = 0; i < NC / 4; ++i) {
        const float4 t = reinterpret_cast<const float4*>(xi)[i];
        v[4 * i] += t.x;
        v[4 * i + 1] += t.y;
        v[4 * i + 2] += t.z;
        v[4 * i + 3] += t.w;
      }
#pragma unroll
      for (int i = 0; i < NC; ++i) v[i] = ok ? v[i] * P.scale : 0.f;
    } else {
#pragma unroll
      for (int i = 0; i < NC; ++i) v[i] = 0.f;
    }
    const int sI = safe_shape(g, P.zone_shape, I, status);
    const BlockBox qb = block_box(g, sI, I);
    const int tok = block_token(g, qb, m);
    if (!g.partial || block_slot_in_grid(g, qb, m))  // a slot outside the grid has no row
      store_row<NC>(P.out0, int64_t(tok) * P.tok_stride + int64_t(head) * D + keep, v, P.out_fp32);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ------------------------------------------------------------ dq, short rows
// The sparse plan's dQ pass (rows of few key blocks on average; every row): a
// row of a few key blocks is mostly fixed cost (the Q / dO copies, the first
// K / V copies, the epilogue), so each CTA takes about half the tensor memory
// and 96 KB of shared memory, two CTAs share an SM, and each loops over the
// rows of its stride with the copies of the next row started as soon as the
// current one frees their buffers.
//   warp 0      copies: per row Q and dO (5-D TMA) into two tiles that are the
//               A operands of the row's S / dP products; per step K and V of
//               the step's two key blocks (5-D TMA from the box origins the
//               block-id prefetch keeps);
//   warp 1      TMEM owner and issuer, per step: S_j = Q [K_j0 K_j1]^T and
//               dP_j = dO [V_j0 V_j1]^T (.ws M=64, N=128, A from shared
//               memory), then, once dS_j is written over S_j's first 32
//               columns, dQ_parts += dS_j K_j (dS as the TMEM A operand);
//   warps 2..5  dS = P (dP - D) with P = exp2(S scale log2e - LSE log2e),
//               one thread per TMEM lane (row m, key block kh of the step),
//               then the epilogue: the key-block parts of dQ added across
//               the lane halves through shared memory (over the V slot, free
//               once the row's last dP has completed), scaled, and stored.
// TMEM: S (dS over its first 32 columns) at 0, dP at 64, the dQ parts at 128.
// Barrier phases run on across rows (steps and rows of the CTA counted from
// 0); every wait is placed so that the phase after the awaited one needs a
// step the waiter has not yet enabled.
constexpr int kDqSmallThreads = 64 + 128;

template <int D>
struct DqSmallSmem {
  static constexpr uint32_t kQ = 0;                      // Q [dh][64][128 B]
  static constexpr uint32_t kDO = D * 128;               // dO
  static constexpr uint32_t kHalf = kKB * D * 128;       // K (or V) of one step, [dh][key block][64][128 B]
  static constexpr uint32_t kK = 2 * D * 128;
  static constexpr uint32_t kV = kK + kHalf;
  static constexpr uint32_t kDesc = kV + kHalf;          // block-id ring
  static constexpr uint32_t kBar = kDesc + kDescRing * 4;
  static constexpr uint32_t kTotal = kBar + 128;
  // epilogue over the V slot: exchange of half rows [lane half][64 rows][kXC + 4 floats] in rounds
  // of kXC channels, then the bf16 dQ tile ([dh][64][128 B], swizzled)
  static constexpr int kXC = D == 128 ? 32 : 16;
  static constexpr uint32_t kXPitch = kXC + 4;
  static_assert(2 * 64 * kXPitch * 4 <= kHalf && D * 128 <= kHalf, "epilogue buffers fit the V slot");
  static_assert(2 * (kTotal + 2048) <= 228 * 1024, "two CTAs per SM");
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kTS = 0, kTP = 64, kTQ = 128;
};

template <int D>
__global__ void __launch_bounds__(kDqSmallThreads, 2) bsa_dq_small_kernel(const __grid_constant__ BwdParams P) {
  using L = DqSmallSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* qd_full = bars + 0;     // Q and dO of the row landed
  uint64_t* qd_free = bars + 1;     // the row's last S / dP products complete (Q, dO tiles free)
  uint64_t* k_full = bars + 2;      // K of the step landed
  uint64_t* v_full = bars + 3;      // V of the step landed
  uint64_t* v_free = bars + 4;      // S / dP of the step complete (V slot free)
  uint64_t* s_full = bars + 5;      // S / dP of the step complete
  uint64_t* ds_full = bars + 6;     // dS of the step written (4 warps)
  uint64_t* b_done = bars + 7;      // dQ product of the step complete (K slot, S / dP columns free)
  uint64_t* dq_free = bars + 8;     // the row's dQ parts read by the epilogue (4 warps)
  uint64_t* stage_free = bars + 9;  // the row's epilogue done with the V slot
  uint64_t* mma_done = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 12);
  const Geo& g = P.g;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = P.status;
  const int rows = P.heads * g.n_blocks;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 11; ++i) mbar_init(&bars[i], (i == 6 || i == 8) ? 4 : 1);
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
  const uint32_t tS = tbase + L::kTS, tP = tbase + L::kTP, tdQ = tbase + L::kTQ;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    IdCache dc{reinterpret_cast<int*>(sm + L::kDesc), 0};
    dc.zone_shape = P.zone_shape;
    bool ok = true;
    int lq = 0, gs = 0, q_iss = 0, k_iss = 0, v_iss = 0;
    for (int row = blockIdx.x; row < rows && ok; row += gridDim.x) {
      int beg;
      const int cnt = bwd_list(P, row, &beg);
      const int nsteps = (cnt + kKB - 1) / kKB;
      if (nsteps == 0) continue;
      const int I = row % g.n_blocks, head = row / g.n_blocks;
      if (lane == 0) {
        // the tiles held the previous row's Q / dO until its last S / dP completed
        if (lq > 0) ok = mbar_wait_abortable(qd_free, (lq - 1) & 1, status, abort_flag);
        if (ok) {
          const int sI = safe_shape(g, P.zone_shape, I, status);
          const BlockBox qb = block_box(g, sI, I);
          mbar_arrive_expect_tx(qd_full, 2 * D * 128);
          for (int dh = 0; dh < D / 64; ++dh) {
            tma_load_5d(sm + L::kQ + dh * kBoxBytes, &P.mq[sI], qd_full, dh * 64, head, qb.w0, qb.h0, qb.t0);
            tma_load_5d(sm + L::kDO + dh * kBoxBytes, &P.mdo[sI], qd_full, dh * 64, head, qb.w0, qb.h0, qb.t0);
          }
          q_iss = lq + 1;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      dc.filled = 0;
      for (int j = 0; j < nsteps && ok; ++j, ++gs) {
        dc.ensure(kKB * j + kKB - 1, g, P.idx, beg, cnt, status, lane);
        int4 bx[kKB];
        for (int slot = 0; slot < kKB; ++slot) bx[slot] = dc.box(kKB * j + slot);
        if (lane == 0) {
          // the K slot last held step gs - 1: free once its dQ product completed
          if (gs > 0) ok = mbar_wait_abortable(b_done, (gs - 1) & 1, status, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(k_full, L::kHalf);
            for (int slot = 0; slot < kKB; ++slot)
              for (int dh = 0; dh < D / 64; ++dh)
                tma_load_5d(sm + L::kK + dh * (kKB * kBoxBytes) + slot * kBoxBytes, &P.mk[bx[slot].x], k_full, dh * 64,
                            head, bx[slot].w, bx[slot].z, bx[slot].y);
            k_iss = gs + 1;
          }
          // the V slot last held step gs - 1 (free once its S / dP completed)
          // and, before a row's first step, the previous row's epilogue
          if (ok && gs > 0) ok = mbar_wait_abortable(v_free, (gs - 1) & 1, status, abort_flag);
          if (ok && j == 0 && lq > 0) ok = mbar_wait_abortable(stage_free, (lq - 1) & 1, status, abort_flag);
          if (ok) {
            mbar_arrive_expect_tx(v_full, L::kHalf);
            for (int slot = 0; slot < kKB; ++slot)
              for (int dh = 0; dh < D / 64; ++dh)
                tma_load_5d(sm + L::kV + dh * (kKB * kBoxBytes) + slot * kBoxBytes, &P.mv[bx[slot].x], v_full, dh * 64,
                            head, bx[slot].w, bx[slot].z, bx[slot].y);
            v_iss = gs + 1;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      ++lq;
    }
    if (lane == 0) {
      // drain: every issued copy has landed before the CTA may exit (one buffer each: the last)
      if (q_iss > 0) mbar_wait(qd_full, (q_iss - 1) & 1, status);
      if (k_iss > 0) mbar_wait(k_full, (k_iss - 1) & 1, status);
      if (v_iss > 0) mbar_wait(v_full, (v_iss - 1) & 1, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(64, 64 * kKB, false, false);
      const uint64_t dQa = sdesc_sw128(smem_u32(sm + L::kQ), 16, 1024);    // Q as A of S
      const uint64_t dDOa = sdesc_sw128(smem_u32(sm + L::kDO), 16, 1024);  // dO as A of dP
      const uint64_t dKb = sdesc_sw128(smem_u32(sm + L::kK), 16, 1024);    // K as B of S
      const uint64_t dVb = sdesc_sw128(smem_u32(sm + L::kV), 16, 1024);    // V as B of dP
      // B of the dQ product = K of the step, MN-major, N = 128: 64 channels of
      // key block 0 then the same channels of key block 1
      const uint32_t idQ = idesc_bf16_f32(64, 128, false, true);
      const uint64_t dKmn = sdesc_sw128(smem_u32(sm + L::kK), kBoxBytes, 1024);
      bool ok = true;
      int lq = 0, gs = 0;
      for (int row = blockIdx.x; row < rows && ok; row += gridDim.x) {
        int beg;
        const int cnt = bwd_list(P, row, &beg);
        const int nsteps = (cnt + kKB - 1) / kKB;
        if (nsteps == 0) continue;
        ok = mbar_wait_abortable(qd_full, lq & 1, status, abort_flag);
        for (int j = 0; j < nsteps && ok; ++j, ++gs) {
          // K and V of the step landed; the previous step's dQ product (which
          // read dS from the S columns) complete
          ok = mbar_wait_abortable(k_full, gs & 1, status, abort_flag) &&
               mbar_wait_abortable(v_full, gs & 1, status, abort_flag) &&
               (gs == 0 || mbar_wait_abortable(b_done, (gs - 1) & 1, status, abort_flag));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ws(tS, dQa + kmajor_step(kk, kBoxBytes), dKb + kmajor_step(kk, kKB * kBoxBytes), idS, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ws(tP, dDOa + kmajor_step(kk, kBoxBytes), dVb + kmajor_step(kk, kKB * kBoxBytes), idS, kk > 0 ? 1u : 0u);
          mma_commit(s_full);
          mma_commit(v_free);
          if (j == nsteps - 1) mma_commit(qd_free);
          // dS written; before a row's first dQ product the previous row's parts read
          ok = mbar_wait_abortable(ds_full, gs & 1, status, abort_flag) &&
               (j > 0 || lq == 0 || mbar_wait_abortable(dq_free, (lq - 1) & 1, status, abort_flag));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              mma_ws_ts(tdQ + c * 64, tS + kk * 8, dKmn + uint64_t((c * kKB * kBoxBytes + kk * 2048) >> 4), idQ,
                        (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(b_done);
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
    constexpr int NC = D / 2;
    int lq = 0, gs = 0;
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
      int beg;
      const int cnt = bwd_list(P, row, &beg);
      const int nsteps = (cnt + kKB - 1) / kKB;
      const int I = row % g.n_blocks, head = row / g.n_blocks;
      const int sI = safe_shape(g, P.zone_shape, I, status);
      const BlockBox qb = block_box(g, sI, I);
      if (nsteps == 0) {
        // no key block: dQ = 0
        if (!g.partial || block_slot_in_grid(g, qb, m)) {
          float z[NC];
#pragma unroll
          for (int i = 0; i < NC; ++i) z[i] = 0.f;
          store_row<NC>(P.out0, int64_t(block_token(g, qb, m)) * P.tok_stride + int64_t(head) * D + kh * NC, z,
                        P.out_fp32);
        }
        continue;
      }
      const float lse2 = P.lse2[size_t(row) * 64 + m];
      const float dm = P.dvec[size_t(row) * 64 + m];
      for (int j = 0; j < nsteps; ++j, ++gs) {
        const bool valid = (j * kKB + kh) < cnt;  // warp-uniform
        // keys of a key block clipped by the grid's edge (read before the wait)
        uint64_t members = ~uint64_t(0);
        if (g.partial && valid) members = key_block_members(g, P.zone_shape, __ldg(P.idx + beg + j * kKB + kh));
        mbar_wait_abortable(s_full, gs & 1, status, abort_flag);
        tc_fence_after();
        uint32_t pk[32];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t rs[32], rp[32];
          tmem_ld32(tS + lane_off + h * 32, rs);
          tmem_ld32(tP + lane_off + h * 32, rp);
          tmem_ld_wait();
          mask_scores32(rs, uint32_t(members >> (32 * h)));  // P = exp2(-inf) = 0 there, hence dS = 0
          if (valid) {
            const float c = P.scale_log2, nl = -lse2;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float p0 = fast_exp2(fmaf(__uint_as_float(rs[2 * i]), c, nl));
              const float p1 = fast_exp2(fmaf(__uint_as_float(rs[2 * i + 1]), c, nl));
              pk[16 * h + i] =
                  pack_bf16x2(p0 * (__uint_as_float(rp[2 * i]) - dm), p1 * (__uint_as_float(rp[2 * i + 1]) - dm));
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[16 * h + i] = 0u;
          }
        }
        // dS over the first 32 columns of S (every S / dP value of this lane was read above)
        tmem_st16(tS + lane_off, pk);
        tmem_st16(tS + lane_off + 16, pk + 16);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      // ---------------------------------------------------------- epilogue
      // the row's last dQ product complete: the dQ parts are final and the V
      // slot is free (every dP of the row completed before it)
      mbar_wait_abortable(b_done, (gs - 1) & 1, status, abort_flag);
      tc_fence_after();
      named_bar_sync(1, 128);
      const bool ok = *abort_flag == 0;
      // this thread holds the key-block-kh part of dQ row m; it keeps channel
      // half kh and hands half kh ^ 1 to the other lane half, kXC channels per round
      float* X = reinterpret_cast<float*>(sm + L::kV);
      float v[NC];
#pragma unroll
      for (int c0 = 0; c0 < NC; c0 += L::kXC) {
        float gv[L::kXC];
        tmem_ld_f<L::kXC>(tdQ + lane_off + (kh ^ 1) * NC + c0, gv);
        tmem_ld_f<L::kXC>(tdQ + lane_off + kh * NC + c0, v + c0);
        if (c0 + L::kXC == NC) {
          // this warp's last read of the dQ parts: the next row's first dQ product may overwrite them
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dq_free);
        }
        float* xo = X + ((kh ^ 1) * 64 + m) * L::kXPitch;
#pragma unroll
        for (int i = 0; i < L::kXC / 4; ++i)
          reinterpret_cast<float4*>(xo)[i] = make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]);
        named_bar_sync(1, 128);
        const float* xi = X + (kh * 64 + m) * L::kXPitch;
#pragma unroll
        for (int i = 0; i < L::kXC / 4; ++i) {
          const float4 t = reinterpret_cast<const float4*>(xi)[i];
          v[c0 + 4 * i] = (v[c0 + 4 * i] + t.x) * P.scale;
          v[c0 + 4 * i + 1] = (v[c0 + 4 * i + 1] + t.y) * P.scale;
          v[c0 + 4 * i + 2] = (v[c0 + 4 * i + 2] + t.z) * P.scale;
          v[c0 + 4 * i + 3] = (v[c0 + 4 * i + 3] + t.w) * P.scale;
        }
        named_bar_sync(1, 128);  // the exchange buffer is free for the next round (and the tile)
      }
#pragma unroll
      for (int i = 0; i < NC; ++i) v[i] = ok ? v[i] : 0.f;
      if (!P.out_fp32) {
        uint8_t* tile = sm + L::kV;
        tile_put_row<NC>(tile, m, kh * NC, v);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (tid == 0) {
          for (int h = 0; h < D / 64; ++h) tma_store_5d(&P.mo0[sI], tile + h * kBoxBytes, h * 64, head, qb.w0, qb.h0, qb.t0);
          bulk_commit_group();
          bulk_wait_group_read0();  // the tile stays valid until read
        }
      } else if (!g.partial || block_slot_in_grid(g, qb, m)) {
        store_row<NC>(P.out0, int64_t(block_token(g, qb, m)) * P.tok_stride + int64_t(head) * D + kh * NC, v, true);
      }
      // the V slot is free for the next row's first V: after the tile was read
      // (tid 0 waited above) or after every thread's last exchange read
      named_bar_sync(1, 128);
      if (tid == 0) mbar_arrive(stage_free);
      ++lq;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, L::kTmemCols);
  }
}

// --------------------------------------------------------------------- dkdv
// K and V of the key block stay in shared memory (the A operands of every
// S^T / dP^T product). Three stages of (Q, dO) for two query blocks, each held
// from its load until the dV/dK products of its step complete. LSE and D of
// the step's two query blocks are copied with the stage (bulk copies counted
// on the stage's barrier) into one of two small buffers, released by the
// softmax warps once read: no global load sits on the softmax warps' path.
// The softmax warps form two groups of four taking alternate steps (group
// j % 2 takes step j), one thread per TMEM lane: the thread in lane m + 64 kh
// holds key row m of S^T_j and dP^T_j against query block kh of the step (64
// values each) and writes P^T and dS^T (bf16) back over the first 32 columns
// of its group's S^T and dP^T buffers. They are the TMEM A operands of the
// dV and dK products, and the .ws lane split makes lane half kh accumulate
// the query-block-kh part of dV and dK: the B operand's two 64-column halves
// are the same 64 channels of dO (or Q) of query block 0 and of query block
// 1. The two parts are added once, in the epilogue.
// Two threads issue the products, each in step order: warp 1 issues
// A_j = (S^T_j = K Q_j^T, dP^T_j = V dO_j^T) into group (j % 2)'s buffers once
// stage j has landed and that group's previous dV/dK products (which read
// P^T / dS^T from the same buffers) have completed; warp 10 issues
// B_j = (dV_parts += P^T_j dO_j, dK_parts += dS^T_j Q_j) once P^T_j / dS^T_j
// are written. While one waits on a barrier the other's products keep the
// tensor pipe busy.
template <int D>
struct DkvSmem {
  static constexpr uint32_t kKV = 0;  // K, V [2][dh][64][128 B], resident
  static constexpr uint32_t kKVBytes = 2 * D * 128;
  static constexpr uint32_t kHalf = kKB * D * 128;  // Q (or dO) of one stage, [dh][query block][64][128 B]
  static constexpr uint32_t kStageBytes = 2 * kHalf;
  static constexpr int kStages = 3;
  static constexpr uint32_t kStage0 = kKVBytes;
  // LSE * log2(e) and D of the step's query blocks, [2 buffers][query block][lse2 64 | D 64] floats
  static constexpr uint32_t kLD0 = kStage0 + kStages * kStageBytes;
  static constexpr uint32_t kLDBytes = kKB * 2 * 64 * 4;
  static constexpr uint32_t kDesc = kLD0 + 2 * kLDBytes;  // block-id ring
  static constexpr uint32_t kBar = kDesc + kDescRing * 4;
  static constexpr uint32_t kTotal = kBar + 256;
  // epilogue exchange of dV / dK part quarters: [dV, dK][kh][group][64 rows][D/4 + 4 floats], over the
  // stages, then the bf16 dK and dV tiles
  static constexpr uint32_t kXPitch = D / 4 + 4;
  static constexpr uint32_t kXTile = (2 * 4 * 64 * kXPitch * 4 + 1023) / 1024 * 1024;
  static_assert(kXTile + 2 * D * 128 <= kStages * kStageBytes, "exchange buffer and tiles fit the stages");
  // allocated without alignment slack: the kernel checks that the dynamic
  // shared memory starts on a 1024-byte boundary
  static_assert(kTotal <= 227 * 1024, "shared-memory budget");
};

template <int D, bool G>
__global__ void __launch_bounds__(kBwdThreads, 1) bsa_dkdv_kernel(const __grid_constant__ BwdParams P) {
  using L = DkvSmem<D>;
  constexpr int NS = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  // the 128-byte-swizzled tiles need 1024-byte alignment and there is no
  // slack to align up: refuse (reported, no access) if the start is off
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(P.status, kDevErrBounds);
    return;
  }
  uint8_t* sm = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* kv_full = bars + 0;
  uint64_t* st_full = bars + 1;   // [3] stage landed (Q, dO, LSE, D)
  uint64_t* st_free = bars + 4;   // [3] B of the stage's step complete
  uint64_t* s_full = bars + 7;    // [2] per group: its A complete
  uint64_t* ps_full = bars + 9;   // [2] per group: its P^T, dS^T written to TMEM (4 warps)
  uint64_t* ps_free = bars + 11;  // [2] per group: its B complete (its S^T / dP^T buffers free)
  uint64_t* ld_free = bars + 13;  // [2] LSE / D buffer read by its group (4 warps)
  uint64_t* mma_done = bars + 15;
  uint64_t* b_done = bars + 16;   // every B product complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 17);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 18);

  const Geo& g = P.g;
  const int J = blockIdx.x, head = blockIdx.y;
  const int col = head * g.n_blocks + J;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* status = P.status;
  const int beg = P.ptr[col];
  int cnt = P.ptr[col + 1] - beg;
  if (cnt < 0 || cnt > g.n_blocks) {
    if (threadIdx.x == 0) atomicOr(status, kDevErrBounds);
    cnt = 0;
  }
  const int nsteps = (cnt + kKB - 1) / kKB;
  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&st_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&ps_full[i], kGroupWarps);
      mbar_init(&ps_free[i], 1);
      mbar_init(&ld_free[i], kGroupWarps);
    }
    mbar_init(mma_done, 1);
    mbar_init(b_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  // TMEM columns: S^T [2 groups x 64] at 0 (P^T over its first 32), dP^T
  // [2 x 64] at 128 (dS^T over its first 32), dV parts at 256, dK parts at
  // 256 + D (D columns each)
  const uint32_t tdV = tbase + 256, tdK = tbase + 256 + D;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (nsteps > 0) {
      IdCache dc{reinterpret_cast<int*>(sm + L::kDesc), 0};
      if (lane == 0) {
        const int sJ = safe_shape(g, P.zone_shape, J, status);
        const BlockBox kb = block_box(g, sJ, J);
        mbar_arrive_expect_tx(kv_full, 2 * D * 128);
        for (int dh = 0; dh < D / 64; ++dh) {
          tma_load_5d(sm + L::kKV + dh * kBoxBytes, &P.mk[sJ], kv_full, dh * 64, head, kb.w0, kb.h0, kb.t0);
          tma_load_5d(sm + L::kKV + D * 128 + dh * kBoxBytes, &P.mv[sJ], kv_full, dh * 64, head, kb.w0, kb.h0,
                      kb.t0);
        }
      }
      if constexpr (G) dc.zone_shape = P.zone_shape;
      bool ok = true;
      int issued = 0;
      for (int j = 0; j < nsteps && ok; ++j) {
        dc.ensure(kKB * j + kKB - 1, g, P.idx, beg, cnt, status, lane);
        int4 bx[kKB] = {};
        if constexpr (G)
          for (int slot = 0; slot < kKB; ++slot) bx[slot] = dc.box(kKB * j + slot);
        if (lane == 0) {
          const int s = j % NS;
          // stage s last held step j - 3: free once its dV / dK products completed
          if (j >= NS) ok = mbar_wait_abortable(&st_free[s], ((j / NS) - 1) & 1, status, abort_flag);
          if (ok) {
            uint8_t* stage = sm + L::kStage0 + s * L::kStageBytes;
            mbar_arrive_expect_tx(&st_full[s], L::kStageBytes + L::kLDBytes);
            for (int slot = 0; slot < kKB; ++slot)
              stream_pair<D, G>(P, P.mq, P.mdo, stage, stage + L::kHalf, slot, head, dc.get(kKB * j + slot),
                                bx[slot], &st_full[s]);
            issued = j + 1;
            // LSE / D buffer j % 2 last held step j - 2: free once its group read it.
            // The copies are issued even after a failed wait (an abort, results
            // discarded) so that the stage's barrier completes.
            ok = mbar_wait_abortable(&ld_free[j & 1], ((j >> 1) & 1) ^ 1, status, abort_flag);
            uint8_t* ldb = sm + L::kLD0 + (j & 1) * L::kLDBytes;
            for (int slot = 0; slot < kKB; ++slot) {
              const size_t ro = (size_t(head) * g.n_blocks + dc.get(kKB * j + slot)) * 64;
              bulk_load(ldb + slot * 512, P.lse2 + ro, 256, &st_full[s]);
              bulk_load(ldb + slot * 512 + 256, P.dvec + ro, 256, &st_full[s]);
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      if (lane == 0) {
        // drain: every issued copy has landed before the CTA may exit
        mbar_wait(kv_full, 0, status);
        for (int i = issued - NS > 0 ? issued - NS : 0; i < issued; ++i)
          mbar_wait(&st_full[i % NS], (i / NS) & 1, status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ A issuer
    if (lane == 0 && nsteps > 0) {
      const uint32_t idS = idesc_bf16_f32(64, 64 * kKB, false, false);
      const uint64_t dKa = sdesc_sw128(smem_u32(sm + L::kKV), 16, 1024);            // K as A of S^T
      const uint64_t dVa = sdesc_sw128(smem_u32(sm + L::kKV + D * 128), 16, 1024);  // V as A of dP^T
      const uint32_t sQ0 = smem_u32(sm + L::kStage0);
      const uint64_t dQ0 = sdesc_sw128(sQ0, 16, 1024);              // Q as B of S^T
      const uint64_t dDO0 = sdesc_sw128(sQ0 + L::kHalf, 16, 1024);  // dO as B of dP^T
      constexpr uint64_t kStageStep = L::kStageBytes >> 4;
      bool ok = mbar_wait_abortable(kv_full, 0, status, abort_flag);
      // A_j into group (j % 2)'s buffers once stage j has landed and that
      // group's previous B (which read P^T / dS^T from them) completed
      for (int j = 0; j < nsteps && ok; ++j) {
        ok = mbar_wait_abortable(&st_full[j % NS], (j / NS) & 1, status, abort_flag) &&
             mbar_wait_abortable(&ps_free[j & 1], ((j >> 1) & 1) ^ 1, status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t st = uint64_t(j % NS) * kStageStep;
        const uint32_t tS = tbase + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ws(tS, dKa + kmajor_step(kk, kBoxBytes), dQ0 + st + kmajor_step(kk, kKB * kBoxBytes), idS,
                 kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ws(tS + 128, dVa + kmajor_step(kk, kBoxBytes), dDO0 + st + kmajor_step(kk, kKB * kBoxBytes), idS,
                 kk > 0 ? 1u : 0u);
        mma_commit(&s_full[j & 1]);
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, status);
    }
  } else if (warp == kIssuerB) {
    // ------------------------------------------------------------ B issuer
    if (lane == 0 && nsteps > 0) {
      // B = dO (or Q) of the step, MN-major, N = 128: 64 channels of query
      // block 0 then the same channels of query block 1 (LBO = the block stride)
      const uint32_t idO = idesc_bf16_f32(64, 128, false, true);
      const uint32_t sQ0 = smem_u32(sm + L::kStage0);
      const uint64_t dQmn0 = sdesc_sw128(sQ0, kBoxBytes, 1024);              // Q as B of dK
      const uint64_t dDOmn0 = sdesc_sw128(sQ0 + L::kHalf, kBoxBytes, 1024);  // dO as B of dV
      constexpr uint64_t kStageStep = L::kStageBytes >> 4;
      bool ok = true;
      // B_j once P^T_j / dS^T_j are written (which implies A_j, hence stage j, complete)
      for (int j = 0; j < nsteps && ok; ++j) {
        ok = mbar_wait_abortable(&ps_full[j & 1], (j >> 1) & 1, status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint64_t st = uint64_t(j % NS) * kStageStep;
        const uint32_t tPT = tbase + (j & 1) * 64, tDST = tPT + 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            mma_ws_ts(tdV + c * 64, tPT + kk * 8, dDOmn0 + st + uint64_t((c * kKB * kBoxBytes + kk * 2048) >> 4),
                      idO, (j > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            mma_ws_ts(tdK + c * 64, tDST + kk * 8, dQmn0 + st + uint64_t((c * kKB * kBoxBytes + kk * 2048) >> 4),
                      idO, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&st_free[j % NS]);
        mma_commit(&ps_free[j & 1]);
      }
      mma_commit(b_done);
      mbar_wait(b_done, 0, status);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 2, grp = sw / kGroupWarps, sp = warp & 3;
    const int Ln = sp * 32 + lane;
    const int m = Ln & 63, kh = Ln >> 6;
    const uint32_t lane_off = uint32_t(sp * 32) << 16;
    int k = 0;  // this group's step count
    for (int j = grp; j < nsteps; j += 2, ++k) {
      const bool valid = (j * kKB + kh) < cnt;  // warp-uniform
      mbar_wait_abortable(&s_full[grp], k & 1, status, abort_flag);
      // the stage's copies (LSE / D included) have landed: A_j read the stage,
      // and the wait makes the copied LSE / D visible to this warp
      mbar_wait_abortable(&st_full[j % NS], (j / NS) & 1, status, abort_flag);
      tc_fence_after();
      // LSE * log2(e) and D of the 64 query rows of query block kh of the step
      const float4* ldp = reinterpret_cast<const float4*>(sm + L::kLD0 + (j & 1) * L::kLDBytes + kh * 512);
      uint32_t pp[32], pd[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t rs[32], rp[32];
        tmem_ld32(tbase + lane_off + grp * 64 + h * 32, rs);
        tmem_ld32(tbase + lane_off + 128 + grp * 64 + h * 32, rp);
        tmem_ld_wait();
        if (valid) {
          const float c = P.scale_log2;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 a = ldp[h * 8 + i], e = ldp[16 + h * 8 + i];
            const float p0 = fast_exp2(fmaf(__uint_as_float(rs[4 * i]), c, -a.x));
            const float p1 = fast_exp2(fmaf(__uint_as_float(rs[4 * i + 1]), c, -a.y));
            const float p2 = fast_exp2(fmaf(__uint_as_float(rs[4 * i + 2]), c, -a.z));
            const float p3 = fast_exp2(fmaf(__uint_as_float(rs[4 * i + 3]), c, -a.w));
            pp[16 * h + 2 * i] = pack_bf16x2(p0, p1);
            pp[16 * h + 2 * i + 1] = pack_bf16x2(p2, p3);
            pd[16 * h + 2 * i] =
                pack_bf16x2(p0 * (__uint_as_float(rp[4 * i]) - e.x), p1 * (__uint_as_float(rp[4 * i + 1]) - e.y));
            pd[16 * h + 2 * i + 1] =
                pack_bf16x2(p2 * (__uint_as_float(rp[4 * i + 2]) - e.z), p3 * (__uint_as_float(rp[4 * i + 3]) - e.w));
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pp[16 * h + i] = pd[16 * h + i] = 0u;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&ld_free[j & 1]);
      // P^T and dS^T over the first 32 columns of the group's S^T and dP^T
      // buffers (every S^T / dP^T value of this lane was read above)
      tmem_st16(tbase + lane_off + grp * 64, pp);
      tmem_st16(tbase + lane_off + grp * 64 + 16, pp + 16);
      tmem_st16(tbase + lane_off + 128 + grp * 64, pd);
      tmem_st16(tbase + lane_off + 128 + grp * 64 + 16, pd + 16);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ps_full[grp]);
    }
    // ---------------------------------------------------------- epilogue
    // this group's last B complete; once both groups are here every product
    // is complete and every copy consumed: the stages hold the exchange buffer
    if (k > 0) mbar_wait_abortable(&ps_free[grp], (k - 1) & 1, status, abort_flag);
    tc_fence_after();
    named_bar_sync(1, 32 * kSoftWarps);
    const bool ok = *abort_flag == 0;
    // This thread holds the query-block-kh parts of dV and dK row m; it keeps
    // channel quarter grp * 2 + kh of each and hands quarter grp * 2 + (kh ^ 1)
    // to the thread of the other lane half.
    constexpr int NC = D / 4;
    const int keep = grp * (D / 2) + kh * NC, give = grp * (D / 2) + (kh ^ 1) * NC;
    float vv[NC], vk[NC];
    float* X = reinterpret_cast<float*>(sm + L::kStage0);
    if (nsteps > 0) {  // uniform; on an abort the values are discarded below
      float gv[NC];
      tmem_ld_f<NC>(tdV + lane_off + give, gv);
      float* xo = X + ((0 * 4 + kh * 2 + grp) * 64 + m) * L::kXPitch;
#pragma unroll
      for (int i = 0; i < NC / 4; ++i)
        reinterpret_cast<float4*>(xo)[i] = make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]);
      tmem_ld_f<NC>(tdK + lane_off + give, gv);
      xo = X + ((1 * 4 + kh * 2 + grp) * 64 + m) * L::kXPitch;
#pragma unroll
      for (int i = 0; i < NC / 4; ++i)
        reinterpret_cast<float4*>(xo)[i] = make_float4(gv[4 * i], gv[4 * i + 1], gv[4 * i + 2], gv[4 * i + 3]);
      tmem_ld_f<NC>(tdV + lane_off + keep, vv);
      tmem_ld_f<NC>(tdK + lane_off + keep, vk);
      named_bar_sync(1, 32 * kSoftWarps);
      const float* xv = X + ((0 * 4 + (kh ^ 1) * 2 + grp) * 64 + m) * L::kXPitch;
      const float* xk = X + ((1 * 4 + (kh ^ 1) * 2 + grp) * 64 + m) * L::kXPitch;
#pragma unroll
      for (int i = 0; i < NC / 4; ++i) {
        const float4 tv = reinterpret_cast<const float4*>(xv)[i];
        const float4 tk = reinterpret_cast<const float4*>(xk)[i];
        vv[4 * i] += tv.x;
        vv[4 * i + 1] += tv.y;
        vv[4 * i + 2] += tv.z;
        vv[4 * i + 3] += tv.w;
        vk[4 * i] += tk.x;
        vk[4 * i + 1] += tk.y;
        vk[4 * i + 2] += tk.z;
        vk[4 * i + 3] += tk.w;
      }
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        vv[i] = ok ? vv[i] : 0.f;
        vk[i] = ok ? vk[i] * P.scale : 0.f;
      }
    } else {
#pragma unroll
      for (int i = 0; i < NC; ++i) vv[i] = vk[i] = 0.f;
    }
    const int sJ = safe_shape(g, P.zone_shape, J, status);
    const BlockBox kb = block_box(g, sJ, J);
    // a key slot outside the grid (a block clipped by the edge) has no row; the
    // query slots outside the grid carry P = 0 (LSE = +inf from the prep pass)
    if (!P.out_fp32 && G) {
      // sparse plan: the dK and dV tiles after the exchange buffer (all in the
      // stages) leave as box stores (the dense plan keeps plain row stores,
      // which do not hold the CTA until a tile is read)
      uint8_t* tk = sm + L::kStage0 + L::kXTile;
      uint8_t* tv = tk + D * 128;
      tile_put_row<NC>(tk, m, keep, vk);
      tile_put_row<NC>(tv, m, keep, vv);
      fence_proxy_async_smem();
      named_bar_sync(1, 32 * kSoftWarps);
      if (warp == 2 && lane == 0) {
        for (int h = 0; h < D / 64; ++h) {
          tma_store_5d(&P.mo0[sJ], tk + h * kBoxBytes, h * 64, head, kb.w0, kb.h0, kb.t0);
          tma_store_5d(&P.mo1[sJ], tv + h * kBoxBytes, h * 64, head, kb.w0, kb.h0, kb.t0);
        }
        bulk_commit_group();
        bulk_wait_group_read0();  // the tiles stay valid until read
      }
    } else if (!g.partial || block_slot_in_grid(g, kb, m)) {
      const int tok = block_token(g, kb, m);
      const int64_t off = int64_t(tok) * P.tok_stride + int64_t(head) * D + keep;
      store_row<NC>(P.out0, off, vk, P.out_fp32);
      store_row<NC>(P.out1, off, vv, P.out_fp32);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// --------------------------------------------------------------------- prep
template <typename T>
__device__ __forceinline__ float dot_chunk(const T* a, const T* b, int n);

template <>
__device__ __forceinline__ float dot_chunk<__nv_bfloat16>(const __nv_bfloat16* a, const __nv_bfloat16* b, int n) {
  float s = 0.f;
  for (int i = 0; i < n; i += 8) {
    const uint4 u = *reinterpret_cast<const uint4*>(a + i);
    const uint4 v = *reinterpret_cast<const uint4*>(b + i);
    const uint32_t x[4] = {u.x, u.y, u.z, u.w}, y[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      s = fmaf(__uint_as_float(x[q] << 16), __uint_as_float(y[q] << 16), s);
      s = fmaf(__uint_as_float(x[q] & 0xFFFF0000u), __uint_as_float(y[q] & 0xFFFF0000u), s);
    }
  }
  return s;
}
template <>
__device__ __forceinline__ float dot_chunk<float>(const float* a, const float* b, int n) {
  float s = 0.f;
  for (int i = 0; i < n; i += 4) {
    const float4 u = *reinterpret_cast<const float4*>(a + i);
    const float4 v = *reinterpret_cast<const float4*>(b + i);
    s = fmaf(u.x, v.x, fmaf(u.y, v.y, fmaf(u.z, v.z, fmaf(u.w, v.w, s))));
  }
  return s;
}

template <typename T>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const Geo g, const int32_t* __restrict__ zone_shape,
                                                       const T* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ o_lo,
                                                       const T* __restrict__ dout,
                                                       int64_t tok_stride, int head_dim, const float* __restrict__ lse,
                                                       float* __restrict__ lse2_blk, float* __restrict__ d_blk,
                                                       int* status) {
  const int b = blockIdx.x, head = blockIdx.y;
  const int r = threadIdx.x >> 2, part = threadIdx.x & 3;
  const int s = safe_shape(g, zone_shape, b, status);
  const BlockBox bb = block_box(g, s, b);
  const int tok = block_token(g, bb, r);
  // a slot outside the grid (a block clipped by the edge) has no token
  const bool in_grid = !g.partial || block_slot_in_grid(g, bb, r);
  const int n = head_dim / 4;
  const int64_t off = int64_t(tok) * tok_stride + int64_t(head) * head_dim + part * n;
  float acc = 0.f;
  if (in_grid) {
    acc = dot_chunk<T>(o + off, dout + off, n);
    // the forward's rounding residual restores O to about 16 bits before the dot
    if constexpr (std::is_same_v<T, __nv_bfloat16>) {
      if (o_lo) acc += dot_chunk<T>(o_lo + off, dout + off, n);
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc += __shfl_xor_sync(0xffffffffu, acc, 2);
  if (part == 0) {
    const size_t at = (size_t(head) * g.n_blocks + b) * 64 + r;
    d_blk[at] = acc;
    const int N = g.T * g.H * g.W;
    // A query with no keys has LSE = -inf and, by definition, P = 0 and no
    // gradient. Storing +inf there makes exp2(s * c - lse2) = exp2(-inf) = 0 in
    // both passes without a per-score test; so does a slot outside the grid.
    const float l = in_grid ? lse[int64_t(head) * N + tok] : -INFINITY;
    lse2_blk[at] = l == -INFINITY ? INFINITY : l * 1.4426950408889634f;
  }
}

// ---------------------------------------------------------------------- CSC
__global__ void __launch_bounds__(256) csc_scatter_kernel(const int32_t* __restrict__ row_ptr,
                                                          const int32_t* __restrict__ col_idx, int heads, int nb,
                                                          uint32_t* __restrict__ tmask, int* status) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (row >= heads * nb) return;
  const int head = row / nb, I = row - head * nb;
  const int words = (nb + 31) >> 5;
  const int b = row_ptr[row], e = row_ptr[row + 1];
  for (int k = b + lane; k < e; k += 32) {
    const int J = col_idx[k];
    if (J < 0 || J >= nb) {
      atomicOr(status, kDevErrBounds);
      continue;
    }
    atomicOr(&tmask[(size_t(head) * nb + J) * words + (I >> 5)], 1u << (I & 31));
  }
}

__global__ void __launch_bounds__(256) popc_rows_kernel(const uint32_t* __restrict__ mask, int rows, int words,
                                                        int32_t* __restrict__ cnt) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (row >= rows) return;
  int c = 0;
  for (int w = lane; w < words; w += 32) c += __popc(mask[size_t(row) * words + w]);
#pragma unroll
  for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) cnt[row] = c;
}

struct BwdWs {
  size_t stage_q, stage_k, stage_v, stage_do, lse2, dvec, tmask, ccnt, cptr, ridx, img0, img1, total;
};

BwdWs bwd_ws_layout(const Geo& g, int heads, int head_dim, prism_dtype dtype, int64_t nnz) {
  WsCarver c;
  BwdWs w{};
  if (dtype == PRISM_FP32) {
    const size_t t = size_t(g.T) * g.H * g.W * heads * head_dim * 2;
    w.stage_q = c.take(t);
    w.stage_k = c.take(t);
    w.stage_v = c.take(t);
    w.stage_do = c.take(t);
  }
  const size_t rows = size_t(heads) * g.n_blocks;
  w.lse2 = c.take(rows * 64 * 4);
  w.dvec = c.take(rows * 64 * 4);
  w.tmask = c.take(rows * ((g.n_blocks + 31) / 32) * 4);
  w.ccnt = c.take(rows * 4);
  w.cptr = c.take((rows + 1) * 4);
  w.ridx = c.take(size_t(nnz > 0 ? nnz : 1) * 4);
  // block images of K and V for the dq pass, then of Q and dO for the dkdv pass
  w.img0 = c.take(block_images_bytes(g, heads, head_dim));
  w.img1 = c.take(block_images_bytes(g, heads, head_dim));
  w.total = c.off;
  return w;
}

}  // namespace

prism_status stage_bf16(const void* src, prism_dtype dtype, int64_t tok_stride, int C, int64_t n_tokens,
                        __nv_bfloat16* dst, cudaStream_t s);

size_t bsa_bwd_ws_bytes(const Geo& g, int heads, int head_dim, prism_dtype dtype, int64_t nnz) {
  return bwd_ws_layout(g, heads, head_dim, dtype, nnz).total;
}

}  // namespace prism

using namespace prism;

namespace prism {
namespace {
template <int D, bool G>
cudaError_t launch_dkdv(const BwdParams& P, dim3 grid, cudaStream_t s) {
  const size_t smem = DkvSmem<D>::kTotal;
  const cudaError_t e = cudaFuncSetAttribute(bsa_dkdv_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  bsa_dkdv_kernel<D, G><<<grid, kBwdThreads, smem, s>>>(P);
  return cudaGetLastError();
}
}  // namespace
}  // namespace prism

extern "C" prism_status prism_bsa_bwd(const prism_geometry* geo, const int32_t* zone_shape, const void* q,
                                      const void* k, const void* v, const void* o, const void* o_lo,
                                      const float* lse, const void* dout, prism_dtype dtype, int32_t heads,
                                      int32_t head_dim,
                                      int64_t tok_stride, float scale, const int32_t* row_ptr,
                                      const int32_t* col_idx, int64_t nnz, void* dq, void* dk, void* dv, void* ws,
                                      size_t ws_bytes, void* stream) {
  Geo g;
  prism_status st = make_geo(geo, &g);
  if (st != PRISM_OK) return st;
  if (!zone_shape || !q || !k || !v || !o || !lse || !dout || !row_ptr || !col_idx || !dq || !dk || !dv)
    return PRISM_ERR_ARG;
  if (dtype != PRISM_BF16 && dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
  if (head_dim != 64 && head_dim != 128) return PRISM_ERR_UNSUPPORTED;
  if (heads < 1 || heads > 65535) return PRISM_ERR_UNSUPPORTED;
  if (tok_stride < int64_t(heads) * head_dim || tok_stride % 8) return PRISM_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return PRISM_ERR_ARG;
  if (nnz < 0 || nnz > int64_t(heads) * g.n_blocks * g.n_blocks) return PRISM_ERR_ARG;
  for (const void* p : {q, k, v, o, o_lo, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                        static_cast<const void*>(dv)})
    if (reinterpret_cast<uintptr_t>(p) % 16) return PRISM_ERR_ARG;
  const BwdWs W = bwd_ws_layout(g, heads, head_dim, dtype, nnz);
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < W.total) return PRISM_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  int* status = ws_status(ws);
  const int64_t N = int64_t(g.T) * g.H * g.W;
  const int C = heads * head_dim;
  const void *qb = q, *kb = k, *vb = v, *dob = dout;
  int64_t in_stride = tok_stride;
  if (dtype == PRISM_FP32) {
    auto* sq = reinterpret_cast<__nv_bfloat16*>(w8 + W.stage_q);
    auto* sk = reinterpret_cast<__nv_bfloat16*>(w8 + W.stage_k);
    auto* sv = reinterpret_cast<__nv_bfloat16*>(w8 + W.stage_v);
    auto* sdo = reinterpret_cast<__nv_bfloat16*>(w8 + W.stage_do);
    if ((st = stage_bf16(q, dtype, tok_stride, C, N, sq, s)) != PRISM_OK) return st;
    if ((st = stage_bf16(k, dtype, tok_stride, C, N, sk, s)) != PRISM_OK) return st;
    if ((st = stage_bf16(v, dtype, tok_stride, C, N, sv, s)) != PRISM_OK) return st;
    if ((st = stage_bf16(dout, dtype, tok_stride, C, N, sdo, s)) != PRISM_OK) return st;
    qb = sq; kb = sk; vb = sv; dob = sdo;
    in_stride = C;
  }
  float* lse2 = reinterpret_cast<float*>(w8 + W.lse2);
  float* dvec = reinterpret_cast<float*>(w8 + W.dvec);
  uint32_t* tmask = reinterpret_cast<uint32_t*>(w8 + W.tmask);
  int32_t* ccnt = reinterpret_cast<int32_t*>(w8 + W.ccnt);
  int32_t* cptr = reinterpret_cast<int32_t*>(w8 + W.cptr);
  int32_t* ridx = reinterpret_cast<int32_t*>(w8 + W.ridx);
  const dim3 grid(g.n_blocks, heads);
  if (dtype == PRISM_BF16)
    bwd_prep_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(g, zone_shape, static_cast<const __nv_bfloat16*>(o),
                                                        static_cast<const __nv_bfloat16*>(o_lo),
                                                        static_cast<const __nv_bfloat16*>(dout), tok_stride, head_dim,
                                                        lse, lse2, dvec, status);
  else
    bwd_prep_kernel<float><<<grid, 256, 0, s>>>(g, zone_shape, static_cast<const float*>(o), nullptr,
                                                static_cast<const float*>(dout), tok_stride, head_dim, lse, lse2,
                                                dvec, status);
  const int rows = heads * g.n_blocks;
  const int words = (g.n_blocks + 31) / 32;
  if (cudaMemsetAsync(tmask, 0, size_t(rows) * words * 4, s) != cudaSuccess) return PRISM_ERR_CUDA;
  csc_scatter_kernel<<<unsigned((int64_t(rows) * 32 + 255) / 256), 256, 0, s>>>(row_ptr, col_idx, heads, g.n_blocks,
                                                                                 tmask, status);
  popc_rows_kernel<<<unsigned((int64_t(rows) * 32 + 255) / 256), 256, 0, s>>>(tmask, rows, words, ccnt);
  if (launch_exclusive_scan(ccnt, rows, cptr, s) != cudaSuccess) return PRISM_ERR_CUDA;
  if (launch_mask_to_lists(tmask, cptr, rows, g.n_blocks, nnz, ridx, status, s) != cudaSuccess) return PRISM_ERR_CUDA;

  BwdParams P;
  std::memset(&P, 0, sizeof(P));
  for (int c = 0; c < g.n_cand; ++c) {
    const int bt = g.cand[c][0], bh = g.cand[c][1], bw = g.cand[c][2];
    if ((st = encode_block_map(&P.mq[c], qb, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
    if ((st = encode_block_map(&P.mk[c], kb, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
    if ((st = encode_block_map(&P.mv[c], vb, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
    if ((st = encode_block_map(&P.mdo[c], dob, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
  }
  P.g = g;
  P.zone_shape = zone_shape;
  P.lse2 = lse2;
  P.dvec = dvec;
  P.status = status;
  P.tok_stride = tok_stride;
  P.scale_log2 = scale * 1.4426950408889634f;
  P.scale = scale;
  P.out_fp32 = dtype == PRISM_FP32;
  P.heads = heads;
  uint8_t* img0 = w8 + W.img0;
  uint8_t* img1 = w8 + W.img1;
  // The plan: with at most kSparseBlocksPerRow kept key blocks per row on
  // average each streamed block is read by few rows (or columns), so the
  // passes gather them through the tensor maps instead of making block
  // images of K, V, Q and dO first. Both plans compute the same result.
  const bool gather = nnz <= int64_t(kSparseBlocksPerRow) * rows;
  // dQ: q-stationary over the CSR, streaming K and V
  if (!gather) {
    if ((st = launch_block_images(g, zone_shape, kb, in_stride, heads, head_dim, img0, status, s)) != PRISM_OK)
      return st;
    if ((st = launch_block_images(g, zone_shape, vb, in_stride, heads, head_dim, img1, status, s)) != PRISM_OK)
      return st;
  }
  P.img0 = img0;
  P.img1 = img1;
  P.ptr = row_ptr;
  P.idx = col_idx;
  P.out0 = dq;
  P.out1 = nullptr;
  if (dtype == PRISM_BF16 && gather)
    for (int c = 0; c < g.n_cand; ++c)
      if ((st = encode_block_map(&P.mo0[c], dq, g, heads, head_dim, tok_stride, g.cand[c][0], g.cand[c][1],
                                 g.cand[c][2])) != PRISM_OK)
        return st;
  if (gather) {
    // rows short on average: the short-row kernel, two CTAs per SM, each looping over its rows
    const dim3 grid_small(unsigned(std::min<int64_t>(rows, 2 * device_sm_count())));
    if (head_dim == 128) {
      const size_t smem = DqSmallSmem<128>::kTotal + 1024;
      if (cudaFuncSetAttribute(bsa_dq_small_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
          cudaSuccess)
        return PRISM_ERR_CUDA;
      bsa_dq_small_kernel<128><<<grid_small, kDqSmallThreads, smem, s>>>(P);
    } else {
      const size_t smem = DqSmallSmem<64>::kTotal + 1024;
      if (cudaFuncSetAttribute(bsa_dq_small_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) !=
          cudaSuccess)
        return PRISM_ERR_CUDA;
      bsa_dq_small_kernel<64><<<grid_small, kDqSmallThreads, smem, s>>>(P);
    }
  } else if (head_dim == 128) {
    const size_t smem = DqSmem<128>::kTotal + 1024;
    if (cudaFuncSetAttribute(bsa_dq_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
      return PRISM_ERR_CUDA;
    bsa_dq_kernel<128><<<grid, kBwdThreads, smem, s>>>(P);
  } else {
    const size_t smem = DqSmem<64>::kTotal + 1024;
    if (cudaFuncSetAttribute(bsa_dq_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
      return PRISM_ERR_CUDA;
    bsa_dq_kernel<64><<<grid, kBwdThreads, smem, s>>>(P);
  }
  if (cudaGetLastError() != cudaSuccess) return PRISM_ERR_CUDA;
  // dK, dV: kv-stationary over the CSC, streaming Q and dO (the images
  // overwrite those of K and V once the dq pass is done: same stream)
  if (!gather) {
    if ((st = launch_block_images(g, zone_shape, qb, in_stride, heads, head_dim, img0, status, s)) != PRISM_OK)
      return st;
    if ((st = launch_block_images(g, zone_shape, dob, in_stride, heads, head_dim, img1, status, s)) != PRISM_OK)
      return st;
  }
  P.ptr = cptr;
  P.idx = ridx;
  P.out0 = dk;
  P.out1 = dv;
  if (dtype == PRISM_BF16 && gather)
    for (int c = 0; c < g.n_cand; ++c) {
      const int bt = g.cand[c][0], bh = g.cand[c][1], bw = g.cand[c][2];
      if ((st = encode_block_map(&P.mo0[c], dk, g, heads, head_dim, tok_stride, bt, bh, bw)) != PRISM_OK) return st;
      if ((st = encode_block_map(&P.mo1[c], dv, g, heads, head_dim, tok_stride, bt, bh, bw)) != PRISM_OK) return st;
    }
  const cudaError_t e = head_dim == 128 ? (gather ? launch_dkdv<128, true>(P, grid, s) : launch_dkdv<128, false>(P, grid, s))
                                        : (gather ? launch_dkdv<64, true>(P, grid, s) : launch_dkdv<64, false>(P, grid, s));
  if (e != cudaSuccess) return PRISM_ERR_CUDA;
  return cuda_status(cudaGetLastError());
}
