// gbsa_bwd.cu -- gradients of the attention output (training).
//
// The GBSA article's overview names training as a use of the operator but
// specifies no backward; this computes the exact gradient of the forward's
// function out = Softmax(scale * Q * K_sparse^T + mask) * V_sparse.  For a
// row with visible keys p, weights P_p = exp(s_p - lse) (lse from the
// forward), output O and incoming gradient dO:
//   dV_p += P_p dO                       D = dO . O (delta_kernel)
//   dS_p  = P_p (dO . V_p - D)
//   dQ   += scale sum_p dS_p K_p         dK_p += scale dS_p Q
// The work follows the forward's work list: its item table (sequence, Q
// block, KV head, rows, positions) and live lists (with duplicates, in list
// order).  One CTA per (item, 128-row tile) walks the item's live blocks;
// dQ of its rows stays in registers and is written once, dK and dV of each
// key are added to fp32 outputs with vector atomics (many tiles read a key).
//
// This first version does its five 128 x 128 x 128 products per block with
// fp32 FMAs from shared memory (16-bit tiles, rows padded to 65 words so
// that the rows a warp reads fall in distinct banks); the tensor-core form
// (tcgen05 products with dK / dV accumulated per KV block) is the next step.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gbsa_internal.cuh"
#include "sm100.cuh"

namespace gbsa {

using namespace sm100;

namespace {

constexpr int kBwdThreads = 256;
constexpr int kRowWords = 65;  // 128 16-bit elements + one padding word per row
constexpr int kTileWords = 128 * kRowWords;
constexpr size_t kBwdSmem = 4 * kTileWords * 4     // Q, dO, K, V (16-bit pairs)
                            + 128 * 128 * 4         // P, then dS (fp32)
                            + 3 * 128 * 4;          // per row: lse (log2 units), delta, position
static_assert(kBwdSmem <= 232448, "shared memory budget");

struct BwdParams {
  const int32_t* meta;
  const uint16_t *q, *k, *v, *out, *dout;
  const float* lse;
  const int32_t* block_table;
  const int64_t* cu_kv;  // TND K/V (block_table unused)
  float *dq, *dk, *dv;   // dq [T][N1][D]; dk, dv compact [num_pages][128][N2][D] or [T_kv][N2][D]
  float* delta;          // [T][N1] scratch
  int32_t* dev_status;
  uint32_t signature;
  int32_t N1, N2, G, T, T_kv, top_k, max_pages, num_pages, tile_tokens, tiles_max;
  int64_t kv_page_stride;  // elements between pages of k and v (paged)
  int32_t win_left;
  float scale, scale_log2;
};

// Two 16-bit elements (one 32-bit word, the lower first) as floats.
template <int kDt>
__device__ __forceinline__ float2 widen2(uint32_t w) {
  if constexpr (kDt == 1) {
    __half2 h;
    memcpy(&h, &w, 4);
    return __half22float2(h);
  } else {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
  }
}

// D[t][h] = sum_d dO[t][h][d] * O[t][h][d] (O and dO in the element type of
// q): one warp per (token, head) row.
template <int kDt>
__global__ void __launch_bounds__(256) delta_kernel(const BwdParams p) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= (int64_t)p.T * p.N1) return;
  const uint2 o = reinterpret_cast<const uint2*>(p.out + row * kHeadDim)[lane];
  const uint2 g = reinterpret_cast<const uint2*>(p.dout + row * kHeadDim)[lane];
  const float2 o0 = widen2<kDt>(o.x), o1 = widen2<kDt>(o.y);
  const float2 g0 = widen2<kDt>(g.x), g1 = widen2<kDt>(g.y);
  float s = o0.x * g0.x + o0.y * g0.y + o1.x * g1.x + o1.y * g1.y;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) p.delta[row] = s;
}

// 128 rows of 128 16-bit elements from global rows at `src(r)` (nullptr: a
// row of zeros) into a padded shared tile.  Whole CTA.
template <typename F>
__device__ __forceinline__ void load_tile(uint32_t* tile, F src) {
  for (int i = threadIdx.x; i < 128 * 16; i += kBwdThreads) {
    const int r = i >> 4, c = i & 15;  // row, 16-byte chunk
    const uint16_t* s = src(r);
    uint4 v = make_uint4(0, 0, 0, 0);
    if (s) v = reinterpret_cast<const uint4*>(s)[c];
    uint32_t* d = tile + r * kRowWords + 4 * c;
    d[0] = v.x;
    d[1] = v.y;
    d[2] = v.z;
    d[3] = v.w;
  }
}

template <int kDt>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_kernel(const BwdParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* sQ = reinterpret_cast<uint32_t*>(smem_raw);
  uint32_t* sG = sQ + kTileWords;  // dO
  uint32_t* sK = sG + kTileWords;
  uint32_t* sV = sK + kTileWords;
  float* sP = reinterpret_cast<float*>(sV + kTileWords);  // [128 rows][128 keys]
  float* sL = sP + 128 * 128;                              // lse * log2(e), -inf: no weight
  float* sD = sL + 128;                                    // delta
  int32_t* sPos = reinterpret_cast<int32_t*>(sD + 128);   // query position

  const int32_t* meta = p.meta;
  if ((uint32_t)meta[H_MAGIC] != kMagic || meta[H_VERSION] != kFormatVersion ||
      (uint32_t)meta[H_SIGNATURE] != p.signature) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && p.dev_status)
      atomicOr(p.dev_status, kDevMetaMismatch);
    return;
  }
  const int32_t item = blockIdx.x / p.tiles_max, s = blockIdx.x % p.tiles_max;
  if (item >= meta[H_NITEMS]) return;
  const int64_t off_item = meta[H_OFF_ITEM], off_list = meta[H_OFF_LIST];
  const int4 ia = *reinterpret_cast<const int4*>(meta + off_item + 8 * (int64_t)item);
  const int4 ic = *reinterpret_cast<const int4*>(meta + off_item + 8 * (int64_t)item + 4);
  const int32_t b = ia.x, n_live = ia.y, n_tiles = ia.z, tok_begin = ia.w;
  const int32_t n_store = ic.x, n_used = ic.y, pos0 = ic.z, ku = ic.w;
  if (s >= n_tiles) return;
  const int32_t kvh = item % p.N2;
  const int32_t rows_in_tile = p.tile_tokens * p.G;

  // rows of this tile: token offset r / G in the tile, head r % G
  // (a token past T, which only inconsistent lengths give, is left alone:
  // the metadata status has flagged them)
  auto row_tok = [&](int r) { return s * p.tile_tokens + r / p.G; };
  auto in_t = [&](int r) { return tok_begin + row_tok(r) < p.T; };
  auto row_valid = [&](int r) { return r < rows_in_tile && row_tok(r) < n_store && in_t(r); };
  auto row_used = [&](int r) { return r < rows_in_tile && row_tok(r) < n_used && in_t(r); };
  auto row_index = [&](int r) {  // (token, head) row of q / dq
    return ((int64_t)(tok_begin + row_tok(r)) * p.N1 + kvh * p.G + r % p.G);
  };
  load_tile(sQ, [&](int r) { return row_used(r) ? p.q + row_index(r) * kHeadDim : nullptr; });
  load_tile(sG, [&](int r) { return row_used(r) ? p.dout + row_index(r) * kHeadDim : nullptr; });
  if (threadIdx.x < 128) {
    const int r = threadIdx.x;
    const bool used = row_used(r);
    const float l = used ? p.lse[row_index(r)] : -INFINITY;
    sL[r] = l * 1.4426950408889634f;
    sD[r] = used ? p.delta[row_index(r)] : 0.f;
    sPos[r] = pos0 + row_tok(r);
  }

  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  // ownership: rows / keys ty + 16 i and tx + 16 j; head-dim pairs tx + 16 j
  float dq[8][8];
#pragma unroll
  for (int i = 0; i < 8; i++)
#pragma unroll
    for (int j = 0; j < 8; j++) dq[i][j] = 0.f;

  const int32_t* list = meta + off_list + (int64_t)item * p.top_k;
  const bool tnd = p.cu_kv != nullptr;
  int32_t bad = 0;
  for (int32_t e = 0; e < n_live; e++) {
    const int32_t lb = list[e] & kEntryLbMask;
    // first row of the block in k / v (rows of N2 * D elements; a page is
    // kv_page_stride elements) and in the compact dk / dv
    int64_t row0, grow0;
    if (tnd) {
      row0 = grow0 = p.cu_kv[b] + (int64_t)lb * kPage;
    } else {
      const int32_t page = lb < p.max_pages ? p.block_table[(int64_t)b * p.max_pages + lb] : -1;
      if (page < 0 || page >= p.num_pages) {  // uniform over the CTA
        bad |= kDevBadPage;
        continue;
      }
      row0 = (int64_t)page * (p.kv_page_stride / ((int64_t)p.N2 * kHeadDim));
      grow0 = (int64_t)page * kPage;
    }
    auto key_ok = [&](int c) {
      const int64_t key = (int64_t)lb * kPage + c;
      return key < ku && (!tnd || row0 + c < p.T_kv);
    };
    __syncthreads();  // the previous block's tiles are no longer read
    load_tile(sK, [&](int c) {
      return key_ok(c) ? p.k + ((row0 + c) * p.N2 + kvh) * kHeadDim : nullptr;
    });
    load_tile(sV, [&](int c) {
      return key_ok(c) ? p.v + ((row0 + c) * p.N2 + kvh) * kHeadDim : nullptr;
    });
    __syncthreads();

    // ---- S and P = exp(s - lse) on visible (row, key) pairs
    {
      float acc[8][8];
#pragma unroll
      for (int i = 0; i < 8; i++)
#pragma unroll
        for (int j = 0; j < 8; j++) acc[i][j] = 0.f;
#pragma unroll 2
      for (int dp = 0; dp < 64; dp++) {
        float2 qv[8], kv[8];
#pragma unroll
        for (int i = 0; i < 8; i++) qv[i] = widen2<kDt>(sQ[(ty + 16 * i) * kRowWords + dp]);
#pragma unroll
        for (int j = 0; j < 8; j++) kv[j] = widen2<kDt>(sK[(tx + 16 * j) * kRowWords + dp]);
#pragma unroll
        for (int i = 0; i < 8; i++)
#pragma unroll
          for (int j = 0; j < 8; j++) acc[i][j] += qv[i].x * kv[j].x + qv[i].y * kv[j].y;
      }
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const int r = ty + 16 * i;
        const int32_t pos = sPos[r];
        const float l2 = sL[r];
#pragma unroll
        for (int j = 0; j < 8; j++) {
          const int c = tx + 16 * j;
          const int32_t key = lb * kPage + c;
          const bool vis = l2 != -INFINITY && key < ku && key <= pos &&
                           (p.win_left < 0 || key >= pos - p.win_left);
          sP[r * 128 + c] = vis ? fast_exp2(acc[i][j] * p.scale_log2 - l2) : 0.f;
        }
      }
    }
    __syncthreads();

    // ---- dV[key][d] += sum_r P[r][key] dO[r][d]   (keys ty + 16 i, d pairs tx + 16 j)
    {
      float2 acc[8][4];
#pragma unroll
      for (int i = 0; i < 8; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = make_float2(0.f, 0.f);
#pragma unroll 2
      for (int r = 0; r < 128; r++) {
        float pv[8];
        float2 gv[4];
#pragma unroll
        for (int i = 0; i < 8; i++) pv[i] = sP[r * 128 + ty + 16 * i];
#pragma unroll
        for (int j = 0; j < 4; j++) gv[j] = widen2<kDt>(sG[r * kRowWords + tx + 16 * j]);
#pragma unroll
        for (int i = 0; i < 8; i++)
#pragma unroll
          for (int j = 0; j < 4; j++) {
            acc[i][j].x += pv[i] * gv[j].x;
            acc[i][j].y += pv[i] * gv[j].y;
          }
      }
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const int c = ty + 16 * i;
        if (!key_ok(c)) continue;
        float* dst = p.dv + ((grow0 + c) * p.N2 + kvh) * kHeadDim;
#pragma unroll
        for (int j = 0; j < 4; j++)
          atomicAdd(reinterpret_cast<float2*>(dst) + tx + 16 * j, acc[i][j]);
      }
    }

    // ---- dS = P (dO . V - delta), in place of P (rows ty + 16 i, keys tx + 16 j)
    {
      float acc[8][8];
#pragma unroll
      for (int i = 0; i < 8; i++)
#pragma unroll
        for (int j = 0; j < 8; j++) acc[i][j] = 0.f;
#pragma unroll 2
      for (int dp = 0; dp < 64; dp++) {
        float2 gv[8], vv[8];
#pragma unroll
        for (int i = 0; i < 8; i++) gv[i] = widen2<kDt>(sG[(ty + 16 * i) * kRowWords + dp]);
#pragma unroll
        for (int j = 0; j < 8; j++) vv[j] = widen2<kDt>(sV[(tx + 16 * j) * kRowWords + dp]);
#pragma unroll
        for (int i = 0; i < 8; i++)
#pragma unroll
          for (int j = 0; j < 8; j++) acc[i][j] += gv[i].x * vv[j].x + gv[i].y * vv[j].y;
      }
      __syncthreads();  // every thread has read P for dV
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const int r = ty + 16 * i;
        const float dlt = sD[r];
#pragma unroll
        for (int j = 0; j < 8; j++) {
          const int c = tx + 16 * j;
          sP[r * 128 + c] = sP[r * 128 + c] * (acc[i][j] - dlt);
        }
      }
    }
    __syncthreads();

    // ---- dQ[r][d] += scale sum_key dS[r][key] K[key][d]   (rows ty + 16 i, d pairs tx + 16 j)
#pragma unroll 2
    for (int c = 0; c < 128; c++) {
      float sv[8];
      float2 kv[4];
#pragma unroll
      for (int i = 0; i < 8; i++) sv[i] = sP[(ty + 16 * i) * 128 + c];
#pragma unroll
      for (int j = 0; j < 4; j++) kv[j] = widen2<kDt>(sK[c * kRowWords + tx + 16 * j]);
#pragma unroll
      for (int i = 0; i < 8; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) {
          dq[i][2 * j] += sv[i] * kv[j].x;
          dq[i][2 * j + 1] += sv[i] * kv[j].y;
        }
    }

    // ---- dK[key][d] += scale sum_r dS[r][key] Q[r][d]   (keys ty + 16 i, d pairs tx + 16 j)
    {
      float2 acc[8][4];
#pragma unroll
      for (int i = 0; i < 8; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = make_float2(0.f, 0.f);
#pragma unroll 2
      for (int r = 0; r < 128; r++) {
        float sv[8];
        float2 qv[4];
#pragma unroll
        for (int i = 0; i < 8; i++) sv[i] = sP[r * 128 + ty + 16 * i];
#pragma unroll
        for (int j = 0; j < 4; j++) qv[j] = widen2<kDt>(sQ[r * kRowWords + tx + 16 * j]);
#pragma unroll
        for (int i = 0; i < 8; i++)
#pragma unroll
          for (int j = 0; j < 4; j++) {
            acc[i][j].x += sv[i] * qv[j].x;
            acc[i][j].y += sv[i] * qv[j].y;
          }
      }
#pragma unroll
      for (int i = 0; i < 8; i++) {
        const int c = ty + 16 * i;
        if (!key_ok(c)) continue;
        float* dst = p.dk + ((grow0 + c) * p.N2 + kvh) * kHeadDim;
#pragma unroll
        for (int j = 0; j < 4; j++)
          atomicAdd(reinterpret_cast<float2*>(dst) + tx + 16 * j,
                    make_float2(acc[i][j].x * p.scale, acc[i][j].y * p.scale));
      }
    }
  }

  // dQ of the tile's stored rows (0 for rows past seqused_q or with no key)
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const int r = ty + 16 * i;
    if (!row_valid(r)) continue;
    float* dst = p.dq + row_index(r) * kHeadDim;
#pragma unroll
    for (int j = 0; j < 4; j++)
      reinterpret_cast<float2*>(dst)[tx + 16 * j] =
          make_float2(dq[i][2 * j] * p.scale, dq[i][2 * j + 1] * p.scale);
  }
  if (bad && p.dev_status) atomicOr(p.dev_status, bad);
}

}  // namespace

size_t backward_smem_bytes() { return kBwdSmem; }

cudaError_t launch_backward(const int32_t* meta, const void* q, const void* k, const void* v,
                            const void* out, const void* dout, const float* lse,
                            const int32_t* block_table, const int64_t* cu_seqlens_kv, float* dq,
                            float* dk, float* dv, size_t dk_bytes, float* delta,
                            int32_t* dev_status, uint32_t signature, int32_t N1, int32_t N2,
                            int32_t T, int32_t T_kv, int32_t top_k, int32_t max_pages,
                            int32_t num_pages, int64_t kv_page_stride, int32_t tile_tokens,
                            int32_t tiles_max, int32_t n_items, int32_t win_left, float scale,
                            int32_t dtype, cudaStream_t stream) {
  BwdParams p;
  p.meta = meta;
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.out = static_cast<const uint16_t*>(out);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.block_table = block_table;
  p.cu_kv = cu_seqlens_kv;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.delta = delta;
  p.dev_status = dev_status;
  p.signature = signature;
  p.N1 = N1;
  p.N2 = N2;
  p.G = N1 / N2;
  p.T = T;
  p.T_kv = T_kv;
  p.top_k = top_k;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.tile_tokens = tile_tokens;
  p.tiles_max = tiles_max;
  p.kv_page_stride = kv_page_stride;
  p.win_left = win_left;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaError_t e;
  if ((e = cudaMemsetAsync(dk, 0, dk_bytes, stream)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dv, 0, dk_bytes, stream)) != cudaSuccess) return e;
  const int64_t rows = (int64_t)T * N1;
  const unsigned dblocks = (unsigned)((rows + 7) / 8);
  auto bwd = dtype == 1 ? bwd_kernel<1> : bwd_kernel<0>;
  static int configured_device = -1;
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (configured_device != dev) {
    for (auto fn : {bwd_kernel<0>, bwd_kernel<1>})
      if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kBwdSmem)) != cudaSuccess)
        return e;
    configured_device = dev;
  }
  {
    NvtxRange range("gbsa_backward");
    if (dtype == 1)
      delta_kernel<1><<<dblocks, 256, 0, stream>>>(p);
    else
      delta_kernel<0><<<dblocks, 256, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd<<<(unsigned)((int64_t)n_items * tiles_max), kBwdThreads, kBwdSmem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace gbsa
