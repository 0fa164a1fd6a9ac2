// Host-side helpers shared by the entry points: argument validation, the
// workspace layout, and TMA descriptor encoding (through the runtime's driver
// entry point, so the library does not link libcuda directly).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "../../include/prism.h"
#include "common.cuh"

namespace prism {

// Bytes reserved at the start of every workspace for the device status word.
constexpr size_t kWsHeader = 256;

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Sequential carve-out of a workspace.
struct WsCarver {
  size_t off = kWsHeader;
  size_t take(size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  }
};

prism_status make_geo(const prism_geometry* geo, Geo* out);
prism_status cuda_status(cudaError_t e);

// Encodes a tiled TMA descriptor. dims/strides follow the driver API
// (strides in bytes for dims 1..rank-1).
prism_status encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                          const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                          CUtensorMapSwizzle swizzle);

// 5-D map over a token-major [N, heads, d] bf16 tensor viewed as
// (d, heads, W, H, T), box (64, 1, bw, bh, bt): one 64-channel slice of one
// head of one block.
prism_status encode_block_map(CUtensorMap* map, const void* base, const Geo& g, int heads, int head_dim,
                              int64_t tok_stride, int bt, int bh, int bw);

inline int* ws_status(void* ws) { return reinterpret_cast<int*>(ws); }

// Block-major operand images of a token-major [N, heads, d] bf16 tensor: for
// every (head, block) the block's 64 rows of that head laid out exactly as a
// shared-memory operand tile, [d/64][64 rows][128 B] with the 128-byte
// swizzle, slots outside the grid zero. One image is d * 128 bytes; images
// are head-major, block-minor. A plain bulk copy of an image into a
// 1024-byte-aligned shared-memory tile gives the tile the tensor cores read.
size_t block_images_bytes(const Geo& g, int heads, int head_dim);
prism_status launch_block_images(const Geo& g, const int32_t* zone_shape, const void* src, int64_t tok_stride,
                                 int heads, int head_dim, void* dst, int* status, cudaStream_t s);

// Exclusive scan of n ints: out[0..n] with out[n] = total (one CTA).
cudaError_t launch_exclusive_scan(const int32_t* in, int n, int32_t* out, cudaStream_t s);
// Expands bitmask rows (ceil(nb/32) words each) into ascending index lists at
// row_ptr offsets, clipped at cap (clipping raises kDevErrCapacity).
cudaError_t launch_mask_to_lists(const uint32_t* mask, const int32_t* row_ptr, int rows, int nb, int64_t cap,
                                 int32_t* idx, int* status, cudaStream_t s);
// Number of SMs of the current device.
int device_sm_count();

// Workspace bytes of each entry point (header included).
size_t zone_shapes_ws_bytes(const Geo& g, int feat_c, prism_dtype feat_dtype, int res_c);
size_t block_select_ws_bytes(int heads, int nb, int d);
size_t bsa_fwd_ws_bytes(const Geo& g, int heads, int head_dim, prism_dtype dtype);
size_t bsa_bwd_ws_bytes(const Geo& g, int heads, int head_dim, prism_dtype dtype, int64_t nnz);

}  // namespace prism
