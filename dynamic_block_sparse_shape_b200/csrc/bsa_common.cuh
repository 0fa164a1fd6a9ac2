// Pieces shared by the block-sparse attention kernels (forward and backward).
//
// Tiles. A 64-token block of one head is gathered by TMA as head_dim/64 boxes
// of (64 channels, 1 head, bw, bh, bt) from the token-major tensor; each box
// lands as 64 rows x 128 bytes with the 128-byte swizzle (8-row atoms of 1 KB),
// rows in raster (t, h, w) order, i.e. the K-major operand layout of tcgen05.
//
// MMA shape. A query block has 64 rows. tcgen05.mma with M = 64 runs at half
// rate, while the weight-stationary form (.ws) with M = 64 uses the full
// 128-lane datapath by splitting N over the two lane halves: accumulator
// element (m, n) of an M=64 x N tile sits at TMEM lane m + 64 * (n >= N/2),
// column n mod N/2. Every product here is .ws M = 64 with fp32 accumulation.
#pragma once
#include "common.cuh"
#include "ptx.cuh"

namespace prism {

constexpr int kBoxBytes = 64 * 128;  // one 64-row x 128-byte swizzled box

// The attention's sparse plan: with at most this many kept key blocks per row
// on average (kept pairs / rows) the forward and backward passes gather their
// streamed blocks through 5-D tensor maps instead of making block images, and
// the short-row kernels take every row.
constexpr int kSparseBlocksPerRow = 32;

__device__ __forceinline__ void mma_ws(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.ws.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Same product with the A operand read from TMEM. For M = 64 the .ws datapath
// reads row m of A from lane m and from lane m + 64, so A must be stored in
// both lane halves; packed bf16 pairs, 8 columns per 16-element K step.
__device__ __forceinline__ void mma_ws_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.ws.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Copies this thread's part of a resident 64-row operand tile ([D/64 boxes]
// [64 rows][128 B], 128-byte swizzle, as TMA writes it) into TMEM as a .ws A
// operand: the thread in TMEM lane L writes row L mod 64, column half `ch`
// (D/4 packed columns) at t_addr = tile column base + lane offset. Tensor-core
// reads of a resident tile then cost no shared-memory bandwidth.
template <int D>
__device__ __forceinline__ void tile_to_tmem_a(const uint8_t* tile, uint32_t t_addr, int m, int ch) {
  constexpr int NW = D / 4;  // packed words per thread
  uint32_t v[NW];
  const int d0 = ch * (D / 2);
  const uint8_t* box = tile + (d0 / 64) * kBoxBytes;
  const int c0 = (d0 % 64) / 8;
#pragma unroll
  for (int c = 0; c < NW / 4; ++c) {
    const uint4 u = *reinterpret_cast<const uint4*>(box + sw128_offset(m, c0 + c));
    v[4 * c] = u.x;
    v[4 * c + 1] = u.y;
    v[4 * c + 2] = u.z;
    v[4 * c + 3] = u.w;
  }
  if constexpr (NW == 32) {
    tmem_st16(t_addr + ch * NW, v);
    tmem_st16(t_addr + ch * NW + 16, v + 16);
  } else {
    tmem_st16(t_addr + ch * NW, v);
  }
  tmem_st_wait();
}

// max(a, b, c) in one instruction (three-input max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// K-step addressing as offsets (16-byte units) added to a base descriptor's
// start-address field (bits 0..13; every address here is below 256 KB, so the
// add never carries out of the field). Issuing threads build one base
// descriptor per buffer and add a compile-time constant per step: the k-th
// 16-element step of a K-major [n_box][rows][128 B] operand whose 64-channel
// boxes sit box_stride bytes apart.
__host__ __device__ constexpr uint64_t kmajor_step(int kstep, uint32_t box_stride) {
  return uint64_t((uint32_t(kstep >> 2) * box_stride + uint32_t(kstep & 3) * 32u) >> 4);
}

__device__ __forceinline__ int safe_shape(const Geo& g, const int32_t* zone_shape, int b, int* status) {
  int s = zone_shape[b / g.bpz];
  if (s < 0 || s >= g.n_cand) {
    atomicOr(status, kDevErrBounds);
    s = 0;
  }
  return s;
}

// Slots of key block b that lie in the grid, as a 64-bit mask over the raster
// slots of its box: all ones unless b's zone is clipped by the grid's edge.
// The TMA copy of a clipped box fills its outside slots with zeros; the
// softmax warps give those keys a score of -inf. A block id out of range
// (reported by the coordinate cache) counts as whole.
__device__ __forceinline__ uint64_t key_block_members(const Geo& g, const int32_t* zone_shape, int b) {
  if (b < 0 || b >= g.n_blocks) return ~uint64_t(0);
  const int z = zone_of_block(g, b);
  if (zone_is_whole(g, z)) return ~uint64_t(0);
  int s = __ldg(zone_shape + z);
  if (s < 0 || s >= g.n_cand) s = 0;
  return block_slot_mask(g, block_box(g, s, b));
}

// Scores of keys outside the grid become -inf: r[i] holds key ch*32 + i.
__device__ __forceinline__ void mask_scores32(uint32_t* r, uint32_t members) {
  if (members != 0xffffffffu) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (!((members >> i) & 1u)) r[i] = 0xff800000u;  // -inf
  }
}

// Entries of the block-id ring below.
constexpr int kDescRing = 64;

// Where a block's 5-D tensor-map box starts, with its candidate shape:
// {shape, t0, h0, w0}.
__device__ __forceinline__ int4 block_box_coords(const Geo& g, const int32_t* zone_shape, int b, int* status) {
  int s = __ldg(zone_shape + b / g.bpz);
  if (s < 0 || s >= g.n_cand) {
    atomicOr(status, kDevErrBounds);
    s = 0;
  }
  const BlockBox bb = block_box(g, s, b);
  return make_int4(s, bb.t0, bb.h0, bb.w0);
}

// Block ids named by a CSR / CSC list, read 32 at a time by a whole warp
// (coalesced list reads) into a shared-memory ring, so the thread that issues
// the copies never waits on a dependent global load. Entry e of a list of
// `cnt` blocks processed `step` (a power of two) per step: e < cnt is the
// list's e-th block; a ragged tail (e >= cnt in the last step) repeats the
// step's first block. An id out of range is reported and replaced by 0. With
// `zone_shape` set, the same warp-wide pass also looks up each block's zone
// shape and box origin (block_box_coords) and keeps it in the register of
// the lane that read the id, so the thread that issues tensor-map copies of
// the blocks has neither a dependent load nor the box arithmetic on its path.
struct IdCache {
  int* ring;  // shared memory, kDescRing entries
  int filled;
  int step = 2;
  const int32_t* zone_shape = nullptr;  // non-null: keep box origins
  int4 mybox = make_int4(0, 0, 0, 0);   // this lane's entry of the latest fill
  // Makes entries [0, e] available; the whole warp must call it.
  __device__ __forceinline__ void ensure(int e, const Geo& g, const int32_t* list, int beg, int cnt, int* status,
                                         int lane) {
    while (e >= filled) {
      const int ee = filled + lane;
      int idx = ee < cnt ? ee : (ee & ~(step - 1));
      if (idx >= cnt) idx = 0;
      int J = list[beg + idx];
      if (J < 0 || J >= g.n_blocks) {
        atomicOr(status, kDevErrBounds);
        J = 0;
      }
      ring[ee % kDescRing] = J;
      if (zone_shape) mybox = block_box_coords(g, zone_shape, J, status);
      __syncwarp();
      filled += 32;
    }
  }
  __device__ __forceinline__ int get(int e) const { return ring[e % kDescRing]; }
  // {shape, t0, h0, w0} of entry e, which must belong to the latest fill
  // (fills are 32-entry aligned: entry e sits in lane e % 32); the whole warp
  // calls it
  __device__ __forceinline__ int4 box(int e) const {
    const int l = e & 31;
    return make_int4(__shfl_sync(0xffffffffu, mybox.x, l), __shfl_sync(0xffffffffu, mybox.y, l),
                     __shfl_sync(0xffffffffu, mybox.z, l), __shfl_sync(0xffffffffu, mybox.w, l));
  }
};

// Byte offset of the operand image of (head, block) in a block-major image
// buffer (one D * 128-byte image per block and head, head-major).
__device__ __forceinline__ size_t image_offset(const Geo& g, int head, int b, int D) {
  return (size_t(head) * g.n_blocks + b) * size_t(D) * 128u;
}

// Store 32 (or 16) fp32 values as bf16 or fp32 at dst (16-byte aligned).
template <int NC>
__device__ __forceinline__ void store_row(void* dst, int64_t off, const float* v, bool fp32) {
  if (fp32) {
    float4* d = reinterpret_cast<float4*>(static_cast<float*>(dst) + off);
#pragma unroll
    for (int i = 0; i < NC / 4; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
  } else {
    uint4* d = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst) + off);
#pragma unroll
    for (int i = 0; i < NC / 8; ++i)
      d[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                        pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
  }
}

// TMEM load of NC (32 or 16) consecutive columns into floats.
template <int NC>
__device__ __forceinline__ void tmem_ld_f(uint32_t taddr, float* v) {
  uint32_t r[NC];
  if constexpr (NC == 32) tmem_ld32(taddr, r);
  else tmem_ld16(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < NC; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace prism
