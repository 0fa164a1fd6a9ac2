// a6: block-sparse attention forward over the selected blocks.
//
// Sol-Attn abstract on the Prism paper page: dynamic sparse attention computes
// only the selected key/value blocks. Prism README, "Overview": the selection
// is per query block (hybrid rule). The attention over the selection is
// exact: an online softmax over the kept 64-token key blocks (FlashAttention
// style), fp32 statistics and accumulators, bf16 operands.
//
// One CTA per (query block I, head). Warp roles:
//   warp 0      TMA producer: Q once; per step the K boxes (3-slot ring) and V
//               boxes (2-slot ring) of two selected key blocks, through 5-D
//               tensor maps (one per block shape);
//   warp 1      TMEM owner and single-thread tcgen05 issuer:
//               S_j = Q K_j^T   (.ws M=64, N=128, K=d)   -> TMEM, 3 buffers
//               O  += P_j V_j   (.ws M=64, N=d,   K=128) -> TMEM
//   warps 2..9  softmax: 256 threads, four per query row (two TMEM lane halves
//               x two column halves, 32 keys each); row maxima are exchanged
//               through shared memory; P_j goes to shared memory as the bf16
//               K-major A operand of the PV product (double-buffered).
// The producer and the issuer never block on one barrier: each polls the
// barriers of every operation it could start next (mbarrier.test_wait) and
// starts whichever is ready, so a late K load does not hold back a ready PV
// product and a K slot is refilled as soon as its S product completes.
// The running max is only moved when it grows by more than 8 (log2 units);
// the final division uses the same stale max, so the result is exact while
// the rare O rescale (TMEM load/scale/store) stays off the common path.
#include <cuda_bf16.h>

#include <cmath>
#include <cstring>

#include "bsa_common.cuh"
#include "host.h"

namespace prism {
namespace {

constexpr int kKB = 2;  // key blocks per step
constexpr int kKSlots = 3;
constexpr int kVSlots = 2;
constexpr int kSBufs = 3;
constexpr int kPBufs = 3;
constexpr int kSoftWarps = 8;
constexpr int kFwdThreads = 64 + 32 * kSoftWarps;
constexpr float kRescaleThreshold = 8.0f;

struct FwdParams {
  CUtensorMap mq[kMaxCand];
  CUtensorMap mk[kMaxCand];
  CUtensorMap mv[kMaxCand];
  Geo g;
  const int32_t* zone_shape;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  void* o;
  float* lse;
  int* status;
  int64_t tok_stride;  // of o, elements
  float scale_log2;
  int out_fp32;
};

template <int D>
struct FwdSmem {
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kQBytes = D * 128;
  static constexpr uint32_t kSlotBytes = kKB * D * 128;  // K (or V) of one step
  static constexpr uint32_t kK0 = kQBytes;
  static constexpr uint32_t kV0 = kK0 + kKSlots * kSlotBytes;
  static constexpr uint32_t kPBytes = kKB * kBoxBytes;
  static constexpr uint32_t kP0 = kV0 + kVSlots * kSlotBytes;
  // P buffers 0 and 1 follow the V ring; buffer 2 reuses the Q tile once Q
  // has been copied into TMEM (d = 128: 16 KB), else its own region.
  static constexpr bool kPInQ = kQBytes >= kPBytes;
  static constexpr uint32_t kP2 = kPInQ ? kQ : kP0 + 2 * kPBytes;
  static constexpr uint32_t kRed = kP0 + (kPInQ ? 2 : 3) * kPBytes;
  static constexpr uint32_t kRedBytes = (2 * 4 * 64 + 4 * 64) * 4;
  static constexpr uint32_t kDesc = kRed + kRedBytes;  // block coordinate ring
  static constexpr uint32_t kBar = kDesc + kDescRing * 16;
  static constexpr uint32_t kTotal = kBar + 256;
  static constexpr uint32_t kTmemCols = 512;  // S: 3 x 64 columns, O at 192, Q (A operand) at 256
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1) bsa_fwd_kernel(const __grid_constant__ FwdParams P) {
  using L = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
  uint64_t* q_full = bars + 0;
  // K and V slots have no "empty" barriers of their own: a K slot is free once
  // the S product that read it has completed (s_full), a V slot once its PV
  // product has (p_free).
  uint64_t* k_full = bars + 1;    // [3]
  uint64_t* v_full = bars + 7;    // [2]
  uint64_t* s_full = bars + 11;   // [3]
  uint64_t* s_free = bars + 14;   // [3]
  uint64_t* p_full = bars + 17;   // [3]
  uint64_t* p_free = bars + 20;   // [3]
  uint64_t* mma_done = bars + 23;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 25);
  uint64_t* qa_full = bars + 26;  // Q copied into TMEM by the softmax warps
  float* red = reinterpret_cast<float*>(sm + L::kRed);
  float* redl = red + 2 * 4 * 64;

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

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kKSlots; ++i) {
      mbar_init(&k_full[i], 1);
    }
    for (int i = 0; i < kVSlots; ++i) {
      mbar_init(&v_full[i], 1);
    }
    for (int i = 0; i < kSBufs; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kSoftWarps);
    }
    for (int i = 0; i < kPBufs; ++i) {
      mbar_init(&p_full[i], kSoftWarps);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(mma_done, 1);
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
  const uint32_t tO = tbase + 192;
  const uint32_t tQ = tbase + 256;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (nsteps > 0) {
      DescCache dc{reinterpret_cast<int4*>(sm + L::kDesc), 0};
      if (lane == 0) {
        const int sI = safe_shape(g, P.zone_shape, I, status);
        const BlockBox qb = block_box(g, sI, I);
        mbar_arrive_expect_tx(q_full, L::kQBytes);
        for (int dh = 0; dh < D / 64; ++dh)
          tma_load_5d(sm + L::kQ + dh * kBoxBytes, &P.mq[sI], q_full, dh * 64, head, qb.w0, qb.h0, qb.t0);
      }
      int kj = 0, vj = 0;
      Watchdog wd;
      wd.reset();
      while (kj < nsteps || vj < nsteps) {
        if (kj < nsteps) dc.ensure(kKB * kj + kKB - 1, g, P.col_idx, beg, cnt, P.zone_shape, status, lane);
        int nk = kj, nv = vj, stop = 0;
        if (lane == 0) {
          bool did = false;
          // a K slot is free once the S product of three steps back is done (its s_full phase)
          if (nk < nsteps && mbar_test(&s_full[nk % kKSlots], ((nk / kKSlots) & 1) ^ 1)) {
            const int ks = nk % kKSlots;
            uint8_t* dst = sm + L::kK0 + ks * L::kSlotBytes;
            mbar_arrive_expect_tx(&k_full[ks], L::kSlotBytes);
            for (int slot = 0; slot < kKB; ++slot) {
              const int4 b = dc.get(kKB * nk + slot);
              for (int dh = 0; dh < D / 64; ++dh)
                tma_load_5d(dst + dh * (kKB * kBoxBytes) + slot * kBoxBytes, &P.mk[b.x], &k_full[ks], dh * 64, head,
                            b.y, b.z, b.w);
            }
            ++nk;
            did = true;
          }
          // a V slot is free once the PV product of two steps back is done (its p_free phase)
          if (nv < nk && (nv < kVSlots || mbar_test(&p_free[(nv - kVSlots) % kPBufs], ((nv - kVSlots) / kPBufs) & 1))) {
            const int vs = nv & 1;
            uint8_t* dst = sm + L::kV0 + vs * L::kSlotBytes;
            mbar_arrive_expect_tx(&v_full[vs], L::kSlotBytes);
            for (int slot = 0; slot < kKB; ++slot) {
              const int4 b = dc.get(kKB * nv + slot);
              for (int dh = 0; dh < D / 64; ++dh)
                tma_load_5d(dst + slot * (D * 128) + dh * kBoxBytes, &P.mv[b.x], &v_full[vs], dh * 64, head, b.y,
                            b.z, b.w);
            }
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
        for (int i = kj - kKSlots > 0 ? kj - kKSlots : 0; i < kj; ++i)
          mbar_wait(&k_full[i % kKSlots], (i / kKSlots) & 1, status);
        for (int i = vj - kVSlots > 0 ? vj - kVSlots : 0; i < vj; ++i)
          mbar_wait(&v_full[i & 1], (i >> 1) & 1, status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nsteps > 0) {
      const uint32_t idS = idesc_bf16_f32(64, 64 * kKB, false, false);
      const uint32_t idO = idesc_bf16_f32(64, D, false, true);
      // base descriptors of slot 0 of each ring; slot i adds i * slot bytes / 16
      const uint64_t dK0 = sdesc_sw128(smem_u32(sm + L::kK0), 16, 1024);
      const uint64_t dV0 = sdesc_sw128(smem_u32(sm + L::kV0), kBoxBytes, 1024);
      const uint64_t dP0 = sdesc_sw128(smem_u32(sm + L::kP0), 16, 1024);
      const uint64_t dP2 = sdesc_sw128(smem_u32(sm + L::kP2), 16, 1024);
      bool ok = mbar_wait_abortable(qa_full, 0, status, abort_flag);
      tc_fence_after();
      int sj = 0, pj = 0;
      Watchdog wd;
      wd.reset();
      while (ok && pj < nsteps) {
        bool did = false;
        if (pj < sj && mbar_test(&p_full[pj % kPBufs], (pj / kPBufs) & 1) &&
            mbar_test(&v_full[pj & 1], (pj >> 1) & 1)) {
          tc_fence_after();
          const int pb = pj % kPBufs;
          const uint64_t dP = pb < 2 ? dP0 + uint64_t(pb * (L::kPBytes >> 4)) : dP2;
          const uint64_t dV = dV0 + uint64_t((pj & 1) * (L::kSlotBytes >> 4));
#pragma unroll
          for (int kk = 0; kk < 64 * kKB / 16; ++kk)
            mma_ws(tO, dP + kmajor_step(kk, kBoxBytes), dV + mnmajor_step(kk, D * 128), idO,
                   (pj > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&p_free[pb]);
          ++pj;
          did = true;
        }
        if (sj < nsteps && mbar_test(&k_full[sj % kKSlots], (sj / kKSlots) & 1) &&
            mbar_test(&s_free[sj % kSBufs], ((sj / kSBufs) & 1) ^ 1)) {
          tc_fence_after();
          const uint64_t dK = dK0 + uint64_t((sj % kKSlots) * (L::kSlotBytes >> 4));
          const uint32_t tS = tbase + (sj % kSBufs) * 64;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ws_ts(tS, tQ + kk * 8, dK + kmajor_step(kk, kKB * kBoxBytes), idS, kk > 0 ? 1u : 0u);
          mma_commit(&s_full[sj % kSBufs]);
          ++sj;
          did = true;
        }
        if (did) wd.reset();
        else if (!wd.ok(status, abort_flag)) break;
      }
      // every MMA this thread issued has completed before TMEM is released
      mma_commit(mma_done);
      mbar_wait(mma_done, 0, status);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 2;
    const int sp = warp & 3;
    const int ch = sw >> 2;
    const int Ln = sp * 32 + lane;
    const int m = Ln & 63, kh = Ln >> 6;
    const int q4 = kh * 2 + ch;
    const uint32_t lane_off = uint32_t(sp * 32) << 16;
    float m_run = -INFINITY, l_part = 0.f;
    if (nsteps > 0) {
      // Q becomes the A operand of every S product: one copy into TMEM
      mbar_wait_abortable(q_full, 0, status, abort_flag);
      tile_to_tmem_a<D>(sm + L::kQ, tQ + lane_off, m, ch);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(qa_full);
    }
    for (int j = 0; j < nsteps; ++j) {
      const int sb = j % kSBufs, pb = j % kPBufs, rb = j & 1;
      mbar_wait_abortable(&s_full[sb], (j / kSBufs) & 1, status, abort_flag);
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tbase + lane_off + sb * 64 + ch * 32, r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      const bool valid = (j * kKB + kh) < cnt;  // warp-uniform: kh is fixed per warp
      float mx = -INFINITY;
      if (valid) {
#pragma unroll
        for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(r[i]));
        mx *= P.scale_log2;  // the scale is positive, so it commutes with the max
      }
      red[(rb * 4 + q4) * 64 + m] = mx;
      named_bar_sync(1, 32 * kSoftWarps);
      const float mb = fmaxf(fmaxf(red[(rb * 4 + 0) * 64 + m], red[(rb * 4 + 1) * 64 + m]),
                             fmaxf(red[(rb * 4 + 2) * 64 + m], red[(rb * 4 + 3) * 64 + m]));
      const float m_new = fmaxf(m_run, mb);
      const bool resc = m_new > m_run + kRescaleThreshold;
      if (__any_sync(0xffffffffu, resc)) {
        const float alpha = resc ? fast_exp2(m_run - m_new) : 1.f;
        if (resc) {
          l_part *= alpha;
          m_run = m_new;
        }
        if (j > 0) {
          // O holds PV_0 .. PV_{j-1}: wait for the last of them, then rescale
          mbar_wait_abortable(&p_free[(j - 1) % kPBufs], ((j - 1) / kPBufs) & 1, status, abort_flag);
          tc_fence_after();
          uint32_t o[32];
          const uint32_t ta = tO + lane_off + ch * (D / 4);
          if constexpr (D == 128) {
            tmem_ld32(ta, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(ta, o);
            tmem_st16(ta + 16, o + 16);
          } else {
            tmem_ld16(ta, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(ta, o);
          }
          tmem_st_wait();
          tc_fence_before();
        }
      }
      uint32_t pk[16];
      if (valid) {  // m_run is finite here: it includes this thread's finite maximum
        const float c = P.scale_log2, nm = -m_run;
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(r[2 * i]), c, nm));
          const float p1 = fast_exp2(fmaf(__uint_as_float(r[2 * i + 1]), c, nm));
          lsum += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        l_part += lsum;
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = 0u;
      }
      if (j >= kPBufs) mbar_wait_abortable(&p_free[pb], ((j / kPBufs) & 1) ^ 1, status, abort_flag);
      uint8_t* pt = sm + (pb < 2 ? L::kP0 + pb * L::kPBytes : L::kP2) + kh * kBoxBytes;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(pt + sw128_offset(m, ch * 4 + q)) =
            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[pb]);
    }
    // ---------------------------------------------------------- epilogue
    if (nsteps > 0)
      mbar_wait_abortable(&p_free[(nsteps - 1) % kPBufs], ((nsteps - 1) / kPBufs) & 1, status, abort_flag);
    tc_fence_after();
    redl[q4 * 64 + m] = l_part;
    named_bar_sync(1, 32 * kSoftWarps);
    const bool ok = *abort_flag == 0;  // uniform: read after the barrier
    const float l = redl[m] + redl[64 + m] + redl[128 + m] + redl[192 + m];
    const float inv = (l > 0.f && ok) ? 1.f / l : 0.f;
    const int sI = safe_shape(g, P.zone_shape, I, status);
    const BlockBox qb = block_box(g, sI, I);
    const int tok = block_token(g, qb, m);
    constexpr int NC = D / 4;
    const int doff = kh * (D / 2) + ch * NC;
    float ov[NC];
    if (nsteps > 0) {
      tmem_ld_f<NC>(tO + lane_off + ch * NC, ov);
#pragma unroll
      for (int i = 0; i < NC; ++i) ov[i] = inv == 0.f ? 0.f : ov[i] * inv;
    } else {
#pragma unroll
      for (int i = 0; i < NC; ++i) ov[i] = 0.f;
    }
    store_row<NC>(P.o, int64_t(tok) * P.tok_stride + int64_t(head) * D + doff, ov, P.out_fp32);
    if (q4 == 0) {
      const int N = g.T * g.H * g.W;
      P.lse[int64_t(head) * N + tok] = (l > 0.f && ok) ? (m_run + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
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

}  // namespace

prism_status stage_bf16(const void* src, prism_dtype dtype, int64_t tok_stride, int C, int64_t n_tokens,
                        __nv_bfloat16* dst, cudaStream_t s) {
  if (dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
  const int64_t total = n_tokens * C / 4;
  to_bf16_kernel<<<unsigned((total + 255) / 256), 256, 0, s>>>(static_cast<const float*>(src), tok_stride, C, n_tokens,
                                                               dst);
  return cuda_status(cudaGetLastError());
}

size_t bsa_fwd_ws_bytes(const Geo& g, int heads, int head_dim, prism_dtype dtype) {
  WsCarver c;
  if (dtype == PRISM_FP32) {
    const size_t t = size_t(g.T) * g.H * g.W * heads * head_dim * 2;
    c.take(t); c.take(t); c.take(t);
  }
  return c.off;
}

}  // namespace prism

using namespace prism;

extern "C" prism_status prism_bsa_fwd(const prism_geometry* geo, const int32_t* zone_shape, const void* q,
                                      const void* k, const void* v, prism_dtype dtype, int32_t heads,
                                      int32_t head_dim, int64_t tok_stride, float scale, const int32_t* row_ptr,
                                      const int32_t* col_idx, void* o, float* lse, void* ws, size_t ws_bytes,
                                      void* stream) {
  Geo g;
  prism_status st = make_geo(geo, &g);
  if (st != PRISM_OK) return st;
  if (!zone_shape || !q || !k || !v || !row_ptr || !col_idx || !o || !lse) return PRISM_ERR_ARG;
  if (dtype != PRISM_BF16 && dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
  if (head_dim != 64 && head_dim != 128) return PRISM_ERR_UNSUPPORTED;
  if (heads < 1 || heads > 65535) return PRISM_ERR_UNSUPPORTED;
  if (tok_stride < int64_t(heads) * head_dim || tok_stride % 8) return PRISM_ERR_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return PRISM_ERR_ARG;
  for (const void* p : {q, k, v, static_cast<const void*>(o)})
    if (reinterpret_cast<uintptr_t>(p) % 16) return PRISM_ERR_ARG;
  const size_t need = bsa_fwd_ws_bytes(g, heads, head_dim, dtype);
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < need) return PRISM_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const void* qb = q;
  const void* kb = k;
  const void* vb = v;
  int64_t in_stride = tok_stride;
  if (dtype == PRISM_FP32) {
    const int64_t N = int64_t(g.T) * g.H * g.W;
    const int C = heads * head_dim;
    WsCarver c;
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
  FwdParams P;
  std::memset(&P, 0, sizeof(P));
  for (int c = 0; c < g.n_cand; ++c) {
    const int bt = g.cand[c][0], bh = g.cand[c][1], bw = g.cand[c][2];
    if ((st = encode_block_map(&P.mq[c], qb, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
    if ((st = encode_block_map(&P.mk[c], kb, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
    if ((st = encode_block_map(&P.mv[c], vb, g, heads, head_dim, in_stride, bt, bh, bw)) != PRISM_OK) return st;
  }
  P.g = g;
  P.zone_shape = zone_shape;
  P.row_ptr = row_ptr;
  P.col_idx = col_idx;
  P.o = o;
  P.lse = lse;
  P.status = ws_status(ws);
  P.tok_stride = tok_stride;
  P.scale_log2 = scale * 1.4426950408889634f;
  P.out_fp32 = dtype == PRISM_FP32;
  const dim3 grid(g.n_blocks, heads);
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
