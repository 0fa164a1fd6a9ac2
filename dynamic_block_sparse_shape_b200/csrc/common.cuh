// Geometry of the zone / block partition, shared by host code and kernels.
//
// Zones tile the (T, H, W) token grid in raster (zt, zh, zw) order. Zone z
// uses one block shape (bt, bh, bw) with bt*bh*bw = 64; its blocks are
// numbered raster over the (Zt/bt, Zh/bh, Zw/bw) sub-grid and the global
// block id is z * blocks_per_zone + local id. Tokens inside a block are
// raster (t, h, w), token id n = (t * H + h) * W + w. (Prism README,
// "Overview": spatiotemporal macro-zones with a tailored block shape each.)
//
// A grid that is not a whole number of zones is tiled as if rounded up: the
// last zone along such an axis, and the block boxes in it, are clipped to the
// grid. A block's members are the slots of its box inside the grid; a box with
// none is an empty block. `partial` is set when any axis is clipped.
#pragma once
#include <cstdint>

namespace prism {

// Error bits written into the device status word (first int of a workspace).
enum : int {
  kDevErrTimeout = 1,   // a bounded wait gave up
  kDevErrBounds = 2,    // an index fell outside its buffer (access skipped)
  kDevErrCapacity = 4,  // a list outgrew its buffer (truncated)
};

constexpr int kMaxCand = 16;
constexpr int kBlockTokens = 64;
constexpr int kMaxZoneTokens = 512;

struct Geo {
  int T, H, W;
  int Zt, Zh, Zw;
  int nzt, nzh, nzw;
  int n_zones, bpz, n_blocks;
  int partial;  // some extent is not a multiple of the zone
  int n_cand;
  int cand[kMaxCand][3];
};

struct BlockBox {
  int t0, h0, w0;  // first token's coordinates
  int bt, bh, bw;  // extents
  int shape;       // candidate index
};

__host__ __device__ __forceinline__ BlockBox block_box(const Geo& g, int shape_idx, int b) {
  const int z = b / g.bpz;
  const int l = b - z * g.bpz;
  const int zt = z / (g.nzh * g.nzw);
  const int zr = z - zt * g.nzh * g.nzw;
  const int zh = zr / g.nzw;
  const int zw = zr - zh * g.nzw;
  BlockBox bb;
  bb.shape = shape_idx;
  bb.bt = g.cand[shape_idx][0];
  bb.bh = g.cand[shape_idx][1];
  bb.bw = g.cand[shape_idx][2];
  const int gh = g.Zh / bb.bh, gw = g.Zw / bb.bw;
  const int lt = l / (gh * gw);
  const int lr = l - lt * gh * gw;
  const int lh = lr / gw;
  const int lw = lr - lh * gw;
  bb.t0 = zt * g.Zt + lt * bb.bt;
  bb.h0 = zh * g.Zh + lh * bb.bh;
  bb.w0 = zw * g.Zw + lw * bb.bw;
  return bb;
}

// Token id of the r-th token (raster inside the block) of a block.
__host__ __device__ __forceinline__ int block_token(const Geo& g, const BlockBox& bb, int r) {
  const int rt = r / (bb.bh * bb.bw);
  const int rr = r - rt * bb.bh * bb.bw;
  const int rh = rr / bb.bw;
  const int rw = rr - rh * bb.bw;
  return ((bb.t0 + rt) * g.H + (bb.h0 + rh)) * g.W + (bb.w0 + rw);
}

__host__ __device__ __forceinline__ int zone_of_block(const Geo& g, int b) { return b / g.bpz; }

// True when the r-th slot (raster inside the box) of a block lies in the grid.
__host__ __device__ __forceinline__ bool block_slot_in_grid(const Geo& g, const BlockBox& bb, int r) {
  const int rt = r / (bb.bh * bb.bw);
  const int rr = r - rt * bb.bh * bb.bw;
  const int rh = rr / bb.bw;
  const int rw = rr - rh * bb.bw;
  return bb.t0 + rt < g.T && bb.h0 + rh < g.H && bb.w0 + rw < g.W;
}

// The box's slots inside the grid as a 64-bit mask (bit r = slot r).
__host__ __device__ __forceinline__ uint64_t block_slot_mask(const Geo& g, const BlockBox& bb) {
  const int vt = g.T - bb.t0 < bb.bt ? (g.T - bb.t0 > 0 ? g.T - bb.t0 : 0) : bb.bt;
  const int vh = g.H - bb.h0 < bb.bh ? (g.H - bb.h0 > 0 ? g.H - bb.h0 : 0) : bb.bh;
  const int vw = g.W - bb.w0 < bb.bw ? (g.W - bb.w0 > 0 ? g.W - bb.w0 : 0) : bb.bw;
  if (vt == bb.bt && vh == bb.bh && vw == bb.bw) return ~uint64_t(0);
  const uint64_t row = vw >= 64 ? ~uint64_t(0) : ((uint64_t(1) << vw) - 1);
  uint64_t m = 0;
  for (int rt = 0; rt < vt; ++rt)
    for (int rh = 0; rh < vh; ++rh) m |= row << ((rt * bb.bh + rh) * bb.bw);
  return m;
}

// Extents of zone z clipped to the grid.
__host__ __device__ __forceinline__ void zone_extents(const Geo& g, int z, int* et, int* eh, int* ew) {
  const int zt = z / (g.nzh * g.nzw), zr = z - zt * g.nzh * g.nzw;
  const int zh = zr / g.nzw, zw = zr - zh * g.nzw;
  *et = g.T - zt * g.Zt < g.Zt ? g.T - zt * g.Zt : g.Zt;
  *eh = g.H - zh * g.Zh < g.Zh ? g.H - zh * g.Zh : g.Zh;
  *ew = g.W - zw * g.Zw < g.Zw ? g.W - zw * g.Zw : g.Zw;
}

// True when zone z lies wholly inside the grid.
__host__ __device__ __forceinline__ bool zone_is_whole(const Geo& g, int z) {
  int et, eh, ew;
  zone_extents(g, z, &et, &eh, &ew);
  return et == g.Zt && eh == g.Zh && ew == g.Zw;
}

}  // namespace prism
