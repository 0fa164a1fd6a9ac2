// Host helpers: geometry validation, status mapping, TMA descriptor encoding,
// and the small entry points (status strings, version, counts, device status).
#include <cstring>
#include <mutex>

#include "host.h"

namespace prism {

prism_status cuda_status(cudaError_t e) { return e == cudaSuccess ? PRISM_OK : PRISM_ERR_CUDA; }

prism_status make_geo(const prism_geometry* geo, Geo* out) {
  if (!geo || !out || !geo->cand) return PRISM_ERR_ARG;
  const prism_dim3 g = geo->grid, z = geo->zone;
  if (g.t <= 0 || g.h <= 0 || g.w <= 0 || z.t <= 0 || z.h <= 0 || z.w <= 0) return PRISM_ERR_SHAPE;
  const int64_t zvol = int64_t(z.t) * z.h * z.w;
  if (zvol % kBlockTokens) return PRISM_ERR_SHAPE;
  if (zvol > kMaxZoneTokens) return PRISM_ERR_UNSUPPORTED;
  if (geo->n_cand < 1 || geo->n_cand > kMaxCand) return PRISM_ERR_ARG;
  const int64_t ntok = int64_t(g.t) * g.h * g.w;
  if (ntok > (int64_t(1) << 30)) return PRISM_ERR_UNSUPPORTED;
  Geo r;
  std::memset(&r, 0, sizeof(r));
  r.T = g.t; r.H = g.h; r.W = g.w;
  r.Zt = z.t; r.Zh = z.h; r.Zw = z.w;
  // zones tile the grid rounded up to whole zones; the last along an axis may be clipped
  r.nzt = (g.t + z.t - 1) / z.t; r.nzh = (g.h + z.h - 1) / z.h; r.nzw = (g.w + z.w - 1) / z.w;
  r.partial = (g.t % z.t) || (g.h % z.h) || (g.w % z.w);
  const int64_t nz = int64_t(r.nzt) * r.nzh * r.nzw;
  if (nz * (zvol / kBlockTokens) >= (int64_t(1) << 31)) return PRISM_ERR_UNSUPPORTED;
  r.n_zones = int(nz);
  r.bpz = int(zvol / kBlockTokens);
  r.n_blocks = r.n_zones * r.bpz;
  r.n_cand = geo->n_cand;
  for (int c = 0; c < geo->n_cand; ++c) {
    const prism_dim3 s = geo->cand[c];
    if (s.t <= 0 || s.h <= 0 || s.w <= 0) return PRISM_ERR_SHAPE;
    if (int64_t(s.t) * s.h * s.w != kBlockTokens) return PRISM_ERR_SHAPE;
    if (z.t % s.t || z.h % s.h || z.w % s.w) return PRISM_ERR_SHAPE;
    r.cand[c][0] = s.t; r.cand[c][1] = s.h; r.cand[c][2] = s.w;
  }
  *out = r;
  return PRISM_OK;
}

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
}
}  // namespace

prism_status encode_tiled(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                          const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                          CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return PRISM_ERR_CUDA;
  if (reinterpret_cast<uintptr_t>(base) % 16) return PRISM_ERR_ARG;
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) {
      s[i] = strides_bytes[i];
      if (s[i] % 16) return PRISM_ERR_ARG;
    }
  }
  CUresult r = g_encode(map, dtype, cuuint32_t(rank), const_cast<void*>(base), d, s, b, e,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PRISM_OK : PRISM_ERR_CUDA;
}

prism_status encode_block_map(CUtensorMap* map, const void* base, const Geo& g, int heads, int head_dim,
                              int64_t tok_stride, int bt, int bh, int bw) {
  const uint64_t es = 2;  // bf16
  uint64_t dims[5] = {uint64_t(head_dim), uint64_t(heads), uint64_t(g.W), uint64_t(g.H), uint64_t(g.T)};
  uint64_t strides[4] = {uint64_t(head_dim) * es, uint64_t(tok_stride) * es, uint64_t(tok_stride) * es * g.W,
                         uint64_t(tok_stride) * es * g.W * g.H};
  uint32_t box[5] = {64, 1, uint32_t(bw), uint32_t(bh), uint32_t(bt)};
  return encode_tiled(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace prism

using namespace prism;

extern "C" const char* prism_status_string(prism_status s) {
  switch (s) {
    case PRISM_OK: return "ok";
    case PRISM_ERR_ARG: return "invalid argument";
    case PRISM_ERR_SHAPE: return "invalid grid/zone/candidate geometry";
    case PRISM_ERR_DTYPE: return "unsupported dtype";
    case PRISM_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PRISM_ERR_CAPACITY: return "col_idx capacity smaller than the number of kept blocks";
    case PRISM_ERR_CUDA: return "CUDA runtime or driver error";
    case PRISM_ERR_TIMEOUT: return "a bounded device wait timed out";
    case PRISM_ERR_DEVICE: return "a device-side index check failed";
    case PRISM_ERR_UNSUPPORTED: return "size outside the implemented range";
  }
  return "unknown status";
}

extern "C" int32_t prism_version(void) { return 100; }

extern "C" prism_status prism_geometry_counts(const prism_geometry* geo, int32_t* n_zones, int32_t* n_blocks) {
  Geo g;
  prism_status st = make_geo(geo, &g);
  if (st != PRISM_OK) return st;
  if (n_zones) *n_zones = g.n_zones;
  if (n_blocks) *n_blocks = g.n_blocks;
  return PRISM_OK;
}

extern "C" prism_status prism_workspace_size(prism_op op, const prism_geometry* geo, int32_t heads,
                                             int32_t head_dim, int32_t feat_c, int32_t res_c, prism_dtype in_dtype,
                                             int64_t nnz, size_t* bytes) {
  if (!bytes) return PRISM_ERR_ARG;
  Geo g;
  prism_status st = make_geo(geo, &g);
  if (st != PRISM_OK) return st;
  if (in_dtype != PRISM_BF16 && in_dtype != PRISM_FP32) return PRISM_ERR_DTYPE;
  switch (op) {
    case PRISM_OP_ZONE_SHAPES:
      if (feat_c < 0 || res_c < 0) return PRISM_ERR_ARG;
      *bytes = zone_shapes_ws_bytes(g, feat_c, in_dtype, res_c);
      return PRISM_OK;
    case PRISM_OP_BLOCK_SELECT:
      if (heads < 1 || head_dim < 1) return PRISM_ERR_ARG;
      *bytes = block_select_ws_bytes(heads, g.n_blocks, head_dim);
      return PRISM_OK;
    case PRISM_OP_BSA_FWD:
      if (heads < 1 || (head_dim != 64 && head_dim != 128)) return PRISM_ERR_ARG;
      *bytes = bsa_fwd_ws_bytes(g, heads, head_dim, in_dtype);
      return PRISM_OK;
    case PRISM_OP_BSA_BWD:
      if (heads < 1 || (head_dim != 64 && head_dim != 128) || nnz < 0) return PRISM_ERR_ARG;
      *bytes = bsa_bwd_ws_bytes(g, heads, head_dim, in_dtype, nnz);
      return PRISM_OK;
  }
  return PRISM_ERR_ARG;
}

extern "C" prism_status prism_check_device_status(void* ws, void* stream) {
  if (!ws) return PRISM_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int h = 0;
  if (cudaMemcpyAsync(&h, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return PRISM_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PRISM_ERR_CUDA;
  if (h != 0 && cudaMemsetAsync(ws, 0, sizeof(int), s) != cudaSuccess) return PRISM_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PRISM_ERR_CUDA;
  if (h & kDevErrTimeout) return PRISM_ERR_TIMEOUT;
  if (h) return PRISM_ERR_DEVICE;
  return PRISM_OK;
}
