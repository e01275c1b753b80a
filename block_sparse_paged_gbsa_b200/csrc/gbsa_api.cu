// gbsa_api.cu -- the C ABI of libgbsa (declared in include/gbsa.h): host
// validation, work-list geometry, TMA tensor maps and kernel launches.
//
// Validation follows the GBSA article (cf-1.com/news/4865651), "Constraints":
// head dim 128 only; KV page size 128 = blockShapeY; GQA with N1 % N2 == 0 and
// N1/N2 <= 128; top_k <= 256; only dim0 of K/V may be strided, with stride0 >=
// 128*N2*D and a multiple of N2*D; empty tensors are rejected; PA_BBND needs
// seqused_kv and a block table; "Mask": only the built-in causal mode.
// Device values are never read here (the article's tiling does not check
// values either); the kernels report them through dev_status.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "../../include/gbsa.h"
#include "gbsa_internal.cuh"

namespace gbsa {
cudaError_t launch_metadata(const MetaParams& p, cudaStream_t stream);
size_t forward_smem_bytes();
cudaError_t launch_forward(const CUtensorMap& map_q, const CUtensorMap& map_k,
                           const CUtensorMap& map_v, int32_t* meta,
                           const int32_t* block_table, const int64_t* cu_seqlens_kv, void* out,
                           float* lse, float* ws_o,
                           float* ws_lse, int32_t* dev_status, uint32_t signature, int32_t N1,
                           int32_t N2, int32_t T, int32_t top_k, int32_t max_pages,
                           int32_t num_pages, int32_t tile_tokens, int32_t rows_per_unit,
                           int32_t win_left, int32_t return_lse, float scale_log2,
                           int32_t num_ctas, int64_t comb_cap, bool one_tile_blocks,
                           int32_t dtype, bool half_softmax, float out_scale,
                           uint64_t wait_limit_ns, cudaStream_t stream);
size_t backward_smem_bytes();
cudaError_t launch_backward(const int32_t* meta, const void* q, const void* k, const void* v,
                            const void* out, const void* dout, const float* lse,
                            const int32_t* block_table, const int64_t* cu_seqlens_kv, float* dq,
                            float* dk, float* dv, size_t dk_bytes, float* delta,
                            int32_t* dev_status, uint32_t signature, int32_t N1, int32_t N2,
                            int32_t T, int32_t T_kv, int32_t top_k, int32_t max_pages,
                            int32_t num_pages, int64_t kv_page_stride, int32_t tile_tokens,
                            int32_t tiles_max, int32_t n_items, int32_t win_left, float scale,
                            int32_t dtype, cudaStream_t stream);
}  // namespace gbsa

using namespace gbsa;

namespace {

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Bound of a pipeline wait in the forward kernel unless the problem sets one.
constexpr uint64_t kDefaultWaitLimitNs = 1000000000ull;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Rules that need no device (metadata_mode: T may be 0 = unknown).
gbsa_status validate(const gbsa_problem* p, bool metadata_mode) {
  if (!p) return GBSA_ERR_INVALID_ARG;
  if (p->B < 1 || p->total_q_blocks < 1 || p->top_k < 1 || p->N1 < 1 || p->N2 < 1 ||
      p->block_x < 1)
    return GBSA_ERR_SHAPE;  // empty tensors are rejected
  if (metadata_mode ? p->T < 0 : p->T < 1) return GBSA_ERR_SHAPE;
  if (p->D != kHeadDim) return GBSA_ERR_UNSUPPORTED;
  if (p->block_y != kPage) return GBSA_ERR_UNSUPPORTED;
  if (p->N1 < p->N2 || p->N1 % p->N2 != 0) return GBSA_ERR_SHAPE;
  if (p->N1 / p->N2 > 128) return GBSA_ERR_UNSUPPORTED;
  if (p->top_k > kMaxTopK) return GBSA_ERR_UNSUPPORTED;
  if (p->mask_mode != 1) return GBSA_ERR_UNSUPPORTED;
  // is_packed_gqa = 0 (one head per tile in the article's scheduling) is
  // accepted and run with the packed tiles: every (token, head) row's
  // softmax is computed on its own, so the packing changes no result
  if (p->is_packed_gqa != 0 && p->is_packed_gqa != 1) return GBSA_ERR_INVALID_ARG;
  if (p->win_left < -1 || p->win_right < -1) return GBSA_ERR_INVALID_ARG;
  if (p->return_lse != 0 && p->return_lse != 1) return GBSA_ERR_INVALID_ARG;
  if (p->has_seqused_q != 0 && p->has_seqused_q != 1) return GBSA_ERR_INVALID_ARG;
  if (p->num_ctas < 0 || p->max_blocks_per_split < 0) return GBSA_ERR_INVALID_ARG;
  if (p->dtype != GBSA_DTYPE_BF16 && p->dtype != GBSA_DTYPE_FP16 &&
      p->dtype != GBSA_DTYPE_FP8_E4M3)
    return GBSA_ERR_INVALID_ARG;
  if (p->dtype == GBSA_DTYPE_FP8_E4M3) {
    for (double s : {p->q_scale, p->k_scale, p->v_scale})
      if (!(s > 0.0) || isinf(s)) return GBSA_ERR_INVALID_ARG;
    // the folded score scale and v_scale must stay finite, normal fp32
    const double sc = p->scale > 0.0 ? p->scale : 1.0 / sqrt((double)p->D);
    const double folded = sc * p->q_scale * p->k_scale;
    if (folded > 1e30 || folded < 1e-30 || p->v_scale > 1e30 || p->v_scale < 1e-30)
      return GBSA_ERR_INVALID_ARG;
  }
  // softmaxPrecision: 0 = fp32 online softmax, 1 = half-precision
  // exponentials with the fp32 rescale and fp32 row sums
  if (p->softmax_precision != 0 && p->softmax_precision != 1) return GBSA_ERR_INVALID_ARG;
  if (!(p->scale >= 0.0) || isinf(p->scale)) return GBSA_ERR_INVALID_ARG;
  if (p->wait_limit_ns < 0) return GBSA_ERR_INVALID_ARG;
  if ((int64_t)p->N2 * p->total_q_blocks > 0x7fffffffLL / (p->top_k + 8)) return GBSA_ERR_SHAPE;
  if (p->kv_layout != GBSA_KV_PAGED && p->kv_layout != GBSA_KV_TND) return GBSA_ERR_INVALID_ARG;
  if (!metadata_mode && p->kv_layout == GBSA_KV_TND) {
    if (p->T_kv < 1) return GBSA_ERR_SHAPE;
  } else if (!metadata_mode) {
    if (p->num_pages < 1 || p->max_pages_per_seq < 1) return GBSA_ERR_SHAPE;
    const int64_t page_elems = (int64_t)kPage * p->N2 * p->D;
    if (p->kv_page_stride < page_elems || p->kv_page_stride % ((int64_t)p->N2 * p->D) != 0)
      return GBSA_ERR_SHAPE;
  }
  return GBSA_OK;
}

gbsa_status resolve_ctas(const gbsa_problem* p, int32_t* ctas) {
  if (p->num_ctas > 0) {
    *ctas = p->num_ctas;
    return GBSA_OK;
  }
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      sms < 1) {
    cudaGetLastError();
    return GBSA_ERR_NO_DEVICE;
  }
  *ctas = sms;
  return GBSA_OK;
}

Geometry make_geometry(const gbsa_problem* p, int32_t ctas) {
  Geometry g;
  g.G = p->N1 / p->N2;
  g.tile_tokens = kTileRows / g.G < p->block_x ? kTileRows / g.G : p->block_x;
  g.tiles_max = (int32_t)cdiv(p->block_x, g.tile_tokens);
  g.n_items = p->N2 * p->total_q_blocks;
  const int64_t units_max = (int64_t)g.n_items * cdiv(g.tiles_max, 2);
  if (p->max_blocks_per_split > 0) {
    const int64_t extra = cdiv(units_max * p->top_k, p->max_blocks_per_split);
    g.unit_cap = units_max + extra;
    g.slot_cap = 2 * extra;
    g.comb_cap = units_max < extra ? units_max : extra;
  } else {
    g.unit_cap = units_max + 4LL * ctas;
    g.slot_cap = 8LL * ctas;
    g.comb_cap = units_max < 4LL * ctas ? units_max : 4LL * ctas;
  }
  g.off_seq = kHeaderWords;
  g.off_item = g.off_seq + 8LL * p->B;
  g.off_list = g.off_item + 8LL * g.n_items;
  g.off_unit = g.off_list + (((int64_t)g.n_items * p->top_k + 3) / 4) * 4;
  g.off_comb = g.off_unit + 4 * g.unit_cap;
  g.total_words = g.off_comb + 4 * g.comb_cap;
  g.rows_per_unit = (g.tiles_max < 2 ? g.tiles_max : 2) * g.tile_tokens * g.G;
  return g;
}

// FNV-1a over the host-known fields the work list depends on.
uint32_t problem_signature(const gbsa_problem* p, int32_t ctas) {
  const int32_t words[13] = {p->B,       p->N1,       p->N2,          p->D,
                             p->block_x, p->total_q_blocks, p->top_k, p->mask_mode,
                             p->win_left, p->win_right, p->has_seqused_q, ctas,
                             p->max_blocks_per_split};
  uint32_t h = 0x811C9DC5u;
  for (int i = 0; i < 13; i++) {
    const uint32_t w = (uint32_t)words[i];
    for (int k = 0; k < 4; k++) {
      h ^= (w >> (8 * k)) & 0xffu;
      h *= 0x01000193u;
    }
  }
  return h;
}

struct Workspace {
  size_t o_bytes, lse_off, total;
};

Workspace workspace_layout(const Geometry& g) {
  Workspace w;
  w.o_bytes = (size_t)g.slot_cap * g.rows_per_unit * kHeadDim * sizeof(float);
  w.lse_off = (w.o_bytes + 255) & ~(size_t)255;
  w.total = w.lse_off + (size_t)g.slot_cap * g.rows_per_unit * sizeof(float);
  return w;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    else
      cudaGetLastError();
  }
  return fn;
}

// Bytes per element of q, k and v.
cuuint64_t elem_bytes(int32_t dtype) { return dtype == GBSA_DTYPE_FP8_E4M3 ? 1 : 2; }

// A box row is 128 B: 64 elements of a 16-bit type or 128 E4M3 codes (the
// 128-byte swizzle span).
cuuint32_t box_inner(int32_t dtype) { return (cuuint32_t)(128 / elem_bytes(dtype)); }

bool encode(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
            const cuuint64_t* strides_bytes, const cuuint32_t* box, int32_t dtype) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint32_t es[4] = {1, 1, 1, 1};
  // E4M3 codes travel as plain bytes
  const CUtensorMapDataType t = dtype == GBSA_DTYPE_FP16       ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                : dtype == GBSA_DTYPE_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                               : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // L2 fills of the box rows' own size: a 16-bit head row is 256 B, an E4M3
  // one 128 B (a 256 B fill would bring in the next head's row as well)
  const CUtensorMapL2promotion promo = dtype == GBSA_DTYPE_FP8_E4M3
                                           ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B
                                           : CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
  return fn(map, t, rank, const_cast<void*>(base), dims, strides_bytes, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

int32_t gbsa_abi_version(void) { return GBSA_ABI_VERSION; }

const char* gbsa_status_string(gbsa_status s) {
  switch (s) {
    case GBSA_OK: return "GBSA_OK";
    case GBSA_ERR_INVALID_ARG: return "GBSA_ERR_INVALID_ARG";
    case GBSA_ERR_UNSUPPORTED: return "GBSA_ERR_UNSUPPORTED";
    case GBSA_ERR_SHAPE: return "GBSA_ERR_SHAPE";
    case GBSA_ERR_ALIGNMENT: return "GBSA_ERR_ALIGNMENT";
    case GBSA_ERR_WORKSPACE_TOO_SMALL: return "GBSA_ERR_WORKSPACE_TOO_SMALL";
    case GBSA_ERR_METADATA_TOO_SMALL: return "GBSA_ERR_METADATA_TOO_SMALL";
    case GBSA_ERR_CUDA: return "GBSA_ERR_CUDA";
    case GBSA_ERR_NO_DEVICE: return "GBSA_ERR_NO_DEVICE";
  }
  return "GBSA_ERR_UNKNOWN";
}

gbsa_status gbsa_metadata_size(const gbsa_problem* problem, size_t* bytes) {
  if (!bytes) return GBSA_ERR_INVALID_ARG;
  gbsa_status st = validate(problem, true);
  if (st != GBSA_OK) return st;
  int32_t ctas;
  if ((st = resolve_ctas(problem, &ctas)) != GBSA_OK) return st;
  const Geometry g = make_geometry(problem, ctas);
  if (g.total_words > 0x7fffffffLL) return GBSA_ERR_SHAPE;
  *bytes = (size_t)g.total_words * sizeof(int32_t);
  return GBSA_OK;
}

gbsa_status gbsa_workspace_size(const gbsa_problem* problem, size_t* bytes) {
  if (!bytes) return GBSA_ERR_INVALID_ARG;
  gbsa_status st = validate(problem, true);
  if (st != GBSA_OK) return st;
  int32_t ctas;
  if ((st = resolve_ctas(problem, &ctas)) != GBSA_OK) return st;
  *bytes = workspace_layout(make_geometry(problem, ctas)).total;
  return GBSA_OK;
}

gbsa_status gbsa_metadata(const gbsa_problem* problem, const gbsa_tensors* t, void* meta,
                          size_t meta_bytes, int32_t* dev_status, void* stream) {
  gbsa_status st = validate(problem, true);
  if (st != GBSA_OK) return st;
  if (!t || !meta || !t->sparse_idx || !t->sparse_count || !t->cu_seqlens_q || !t->seqused_kv ||
      (problem->has_seqused_q && !t->seqused_q))
    return GBSA_ERR_INVALID_ARG;
  if (!aligned16(meta)) return GBSA_ERR_ALIGNMENT;
  int32_t ctas;
  if ((st = resolve_ctas(problem, &ctas)) != GBSA_OK) return st;
  const Geometry g = make_geometry(problem, ctas);
  if (g.total_words > 0x7fffffffLL) return GBSA_ERR_SHAPE;
  if (meta_bytes < (size_t)g.total_words * sizeof(int32_t)) return GBSA_ERR_METADATA_TOO_SMALL;
  MetaParams p;
  p.B = problem->B;
  p.T = problem->T;
  p.N1 = problem->N1;
  p.N2 = problem->N2;
  p.block_x = problem->block_x;
  p.total_q_blocks = problem->total_q_blocks;
  p.top_k = problem->top_k;
  p.win_left = problem->win_left;
  p.win_right = problem->win_right;
  p.has_seqused_q = problem->has_seqused_q;
  p.num_ctas = ctas;
  p.forced_split = problem->max_blocks_per_split;
  p.signature = problem_signature(problem, ctas);
  p.geo = g;
  p.sparse_idx = t->sparse_idx;
  p.sparse_count = t->sparse_count;
  p.cu_seqlens_q = t->cu_seqlens_q;
  p.seqused_q = problem->has_seqused_q ? t->seqused_q : nullptr;
  p.seqused_kv = t->seqused_kv;
  p.meta = static_cast<int32_t*>(meta);
  p.dev_status = dev_status;
  NvtxRange range("gbsa_metadata");
  if (launch_metadata(p, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return GBSA_ERR_CUDA;
  }
  return GBSA_OK;
}

gbsa_status gbsa_forward(const gbsa_problem* problem, const gbsa_tensors* t, void* meta,
                         void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
  gbsa_status st = validate(problem, false);
  if (st != GBSA_OK) return st;
  const bool tnd = problem->kv_layout == GBSA_KV_TND;
  if (!t || !meta || !t->q || !t->k || !t->v || !t->sparse_idx || !t->sparse_count ||
      !t->cu_seqlens_q || !t->seqused_kv || !t->out || (tnd ? !t->cu_seqlens_kv : !t->block_table) ||
      (problem->return_lse && !t->lse) || (problem->has_seqused_q && !t->seqused_q))
    return GBSA_ERR_INVALID_ARG;
  if (!aligned16(t->q) || !aligned16(t->k) || !aligned16(t->v) || !aligned16(t->out) ||
      !aligned16(meta) || (t->lse && (reinterpret_cast<uintptr_t>(t->lse) & 3u)))
    return GBSA_ERR_ALIGNMENT;
  int32_t ctas;
  if ((st = resolve_ctas(problem, &ctas)) != GBSA_OK) return st;
  const Geometry g = make_geometry(problem, ctas);
  const Workspace wl = workspace_layout(g);
  if (ws_bytes < wl.total || (wl.total > 0 && (!workspace || !aligned16(workspace))))
    return GBSA_ERR_WORKSPACE_TOO_SMALL;

  const cuuint64_t D = kHeadDim, es = elem_bytes(problem->dtype);
  const cuuint32_t bx = box_inner(problem->dtype);
  CUtensorMap map_q, map_k, map_v;
  {
    const cuuint64_t dims[3] = {D, (cuuint64_t)problem->N1, (cuuint64_t)problem->T};
    const cuuint64_t strides[2] = {D * es, (cuuint64_t)problem->N1 * D * es};
    const cuuint32_t box[3] = {bx, (cuuint32_t)g.G, (cuuint32_t)g.tile_tokens};
    if (!encode(&map_q, t->q, 3, dims, strides, box, problem->dtype)) return GBSA_ERR_CUDA;
  }
  if (tnd) {
    // rows of [T_kv, N2, D]; a box is 128 rows of one head (rows past T_kv read as 0)
    const cuuint64_t dims[3] = {D, (cuuint64_t)problem->N2, (cuuint64_t)problem->T_kv};
    const cuuint64_t strides[2] = {D * es, (cuuint64_t)problem->N2 * D * es};
    const cuuint32_t box[3] = {bx, 1, (cuuint32_t)kPage};
    if (!encode(&map_k, t->k, 3, dims, strides, box, problem->dtype)) return GBSA_ERR_CUDA;
    if (!encode(&map_v, t->v, 3, dims, strides, box, problem->dtype)) return GBSA_ERR_CUDA;
  } else {
    const cuuint64_t dims[4] = {D, (cuuint64_t)problem->N2, (cuuint64_t)kPage,
                                (cuuint64_t)problem->num_pages};
    const cuuint64_t strides[3] = {D * es, (cuuint64_t)problem->N2 * D * es,
                                   (cuuint64_t)problem->kv_page_stride * es};
    const cuuint32_t box[4] = {bx, 1, (cuuint32_t)kPage, 1};
    if (!encode(&map_k, t->k, 4, dims, strides, box, problem->dtype)) return GBSA_ERR_CUDA;
    if (!encode(&map_v, t->v, 4, dims, strides, box, problem->dtype)) return GBSA_ERR_CUDA;
  }
  const bool fp8 = problem->dtype == GBSA_DTYPE_FP8_E4M3;
  double scale = problem->scale > 0.0 ? problem->scale : 1.0 / sqrt((double)problem->D);
  if (fp8) scale *= problem->q_scale * problem->k_scale;  // dequantization folds into the scores
  float* ws_o = static_cast<float*>(workspace);
  float* ws_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + wl.lse_off);
  const cudaError_t e = launch_forward(
      map_q, map_k, map_v, static_cast<int32_t*>(meta), tnd ? nullptr : t->block_table,
      tnd ? t->cu_seqlens_kv : nullptr, t->out,
      problem->return_lse ? t->lse : nullptr, ws_o, ws_lse, dev_status,
      problem_signature(problem, ctas), problem->N1, problem->N2, problem->T, problem->top_k,
      problem->max_pages_per_seq, problem->num_pages, g.tile_tokens, g.rows_per_unit,
      problem->win_left, problem->return_lse, (float)(scale * 1.4426950408889634), ctas,
      g.comb_cap, g.tiles_max == 1, problem->dtype, problem->softmax_precision == 1,
      fp8 ? (float)problem->v_scale : 1.f,
      problem->wait_limit_ns > 0 ? (uint64_t)problem->wait_limit_ns : kDefaultWaitLimitNs,
      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GBSA_ERR_CUDA;
  }
  return GBSA_OK;
}

gbsa_status gbsa_backward_workspace_size(const gbsa_problem* problem, size_t* bytes) {
  if (!bytes) return GBSA_ERR_INVALID_ARG;
  const gbsa_status st = validate(problem, false);
  if (st != GBSA_OK) return st;
  *bytes = (size_t)(((int64_t)problem->T * problem->N1 * 4 + 15) / 16 * 16);
  return GBSA_OK;
}

gbsa_status gbsa_backward(const gbsa_problem* problem, const gbsa_tensors* t, const void* dout,
                          const void* meta, float* dq, float* dk, float* dv, void* workspace,
                          size_t ws_bytes, int32_t* dev_status, void* stream) {
  gbsa_status st = validate(problem, false);
  if (st != GBSA_OK) return st;
  if (problem->dtype == GBSA_DTYPE_FP8_E4M3) return GBSA_ERR_UNSUPPORTED;
  const bool tnd = problem->kv_layout == GBSA_KV_TND;
  if (!t || !meta || !dout || !dq || !dk || !dv || !t->q || !t->k || !t->v || !t->out || !t->lse ||
      !t->sparse_idx || !t->sparse_count || !t->cu_seqlens_q || !t->seqused_kv ||
      (tnd ? !t->cu_seqlens_kv : !t->block_table) || (problem->has_seqused_q && !t->seqused_q))
    return GBSA_ERR_INVALID_ARG;
  if (!aligned16(t->q) || !aligned16(t->k) || !aligned16(t->v) || !aligned16(t->out) ||
      !aligned16(dout) || !aligned16(meta) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv) || (reinterpret_cast<uintptr_t>(t->lse) & 3u))
    return GBSA_ERR_ALIGNMENT;
  size_t need = 0;
  if ((st = gbsa_backward_workspace_size(problem, &need)) != GBSA_OK) return st;
  if (ws_bytes < need || !workspace || !aligned16(workspace)) return GBSA_ERR_WORKSPACE_TOO_SMALL;
  int32_t ctas;
  if ((st = resolve_ctas(problem, &ctas)) != GBSA_OK) return st;
  const Geometry g = make_geometry(problem, ctas);
  const int64_t kv_rows = tnd ? (int64_t)problem->T_kv : (int64_t)problem->num_pages * kPage;
  const size_t dk_bytes = (size_t)(kv_rows * problem->N2 * kHeadDim) * sizeof(float);
  const double scale = problem->scale > 0.0 ? problem->scale : 1.0 / sqrt((double)problem->D);
  const cudaError_t e = launch_backward(
      static_cast<const int32_t*>(meta), t->q, t->k, t->v, t->out, dout, t->lse,
      tnd ? nullptr : t->block_table, tnd ? t->cu_seqlens_kv : nullptr, dq, dk, dv, dk_bytes,
      static_cast<float*>(workspace), dev_status, problem_signature(problem, ctas), problem->N1,
      problem->N2, problem->T, tnd ? problem->T_kv : 0, problem->top_k,
      problem->max_pages_per_seq, problem->num_pages, tnd ? 0 : problem->kv_page_stride,
      g.tile_tokens, g.tiles_max, g.n_items, problem->win_left, (float)scale, problem->dtype,
      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return GBSA_ERR_CUDA;
  }
  return GBSA_OK;
}

}  // extern "C"
