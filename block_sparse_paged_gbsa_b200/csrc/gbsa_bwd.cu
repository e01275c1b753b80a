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
// The five 128 x 128 x 128 products per block run on the tensor cores as
// warp-level mma.sync (m16n8k16, fp32 accumulators) fed by ldmatrix from
// padded shared tiles; P and dS enter them in the element type of q.  Each
// of the 8 warps owns a 32 x 64 tile of every product.  (The tcgen05 form,
// with dK / dV accumulated per KV block in TMEM, is the next step.)
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

constexpr int kBwdThreads = 256;  // 8 warps, each a 32 x 64 tile of every product
// 16-bit tiles of 128 rows x 128 elements; rows padded to 136 elements (272 B)
// so that the 8 rows an ldmatrix reads start in distinct bank groups
constexpr int kRowElems = 136;
constexpr int kTileElems = 128 * kRowElems;
static_assert(128 * 16 % kBwdThreads == 0, "whole 16-byte chunks per thread");
constexpr size_t kBwdSmem = 6 * kTileElems * 2  // Q, dO, K, V, P, dS
                            + 3 * 128 * 4;      // per row: lse (log2 units), delta, position
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

// Two tiles of 128 rows x 128 16-bit elements from global rows at `src0(r)`
// and `src1(r)` (nullptr: a row of zeros) into padded shared tiles (row
// stride kRowElems).  Whole CTA; every thread issues all 16 of its loads
// before its first store, so their latencies overlap.
constexpr int kChunksPerThread = 128 * 16 / kBwdThreads;  // 16-byte chunks of a tile
template <typename F0, typename F1>
__device__ __forceinline__ void load_tiles(uint16_t* t0, uint16_t* t1, F0 src0, F1 src1) {
  uint4 v0[kChunksPerThread], v1[kChunksPerThread];
#pragma unroll
  for (int it = 0; it < kChunksPerThread; it++) {
    const int i = threadIdx.x + it * kBwdThreads;
    const int r = i >> 4, c = i & 15;  // row, 16-byte chunk
    const uint16_t* a = src0(r);
    const uint16_t* b = src1(r);
    v0[it] = a ? reinterpret_cast<const uint4*>(a)[c] : make_uint4(0, 0, 0, 0);
    v1[it] = b ? reinterpret_cast<const uint4*>(b)[c] : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int it = 0; it < kChunksPerThread; it++) {
    const int i = threadIdx.x + it * kBwdThreads;
    const int r = i >> 4, c = i & 15;
    *reinterpret_cast<uint4*>(t0 + r * kRowElems + 8 * c) = v0[it];
    *reinterpret_cast<uint4*>(t1 + r * kRowElems + 8 * c) = v1[it];
  }
}

// 16 bytes global -> shared without registers (zero-filled past src_bytes)
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const uint16_t* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const uint16_t* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

// D += A B for one m16 n8 k16 tile, fp32 accumulators.
template <int kDt>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (kDt == 1)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One warp's 32 x 64 tile of C = A B over K = 128, from shared 16-bit
// tiles with row stride kRowElems:
//   A: kATrans ? stored [k][m] (A = stored^T) : stored [m][k];
//   B: kBTrans ? stored [k][n]               : stored [n][k] (B = stored^T).
// The warp's rows are m0 .. m0 + 31, its columns n0 .. n0 + 63;
// acc[tm][tn] is the m16 n8 fragment at (m0 + 16 tm, n0 + 8 tn).
template <int kDt, bool kATrans, bool kBTrans>
__device__ __forceinline__ void warp_gemm(float (&acc)[2][8][4], const uint16_t* A,
                                          const uint16_t* B, int m0, int n0) {
  const int lane = threadIdx.x & 31;
  const int i8 = lane >> 3, j8 = lane & 7;
#pragma unroll 1
  for (int k0 = 0; k0 < 128; k0 += 16) {
    uint32_t a[2][4];
#pragma unroll
    for (int tm = 0; tm < 2; tm++) {
      const int mb = m0 + 16 * tm;
      if constexpr (kATrans)  // matrices (m, k), (m+8, k), (m, k+8), (m+8, k+8)
        ldsm_x4_t(a[tm], A + (k0 + (i8 >> 1) * 8 + j8) * kRowElems + mb + (i8 & 1) * 8);
      else
        ldsm_x4(a[tm], A + (mb + (lane & 15)) * kRowElems + k0 + (lane >> 4) * 8);
    }
#pragma unroll
    for (int tp = 0; tp < 4; tp++) {  // pairs of n8 tiles
      const int nb = n0 + 16 * tp;
      uint32_t b[4];  // b0, b1 of tile nb, then of tile nb + 8
      if constexpr (kBTrans)  // matrices (k, n), (k+8, n), (k, n+8), (k+8, n+8)
        ldsm_x4_t(b, B + (k0 + (i8 & 1) * 8 + j8) * kRowElems + nb + (i8 >> 1) * 8);
      else
        ldsm_x4(b, B + (nb + (i8 >> 1) * 8 + j8) * kRowElems + k0 + (i8 & 1) * 8);
#pragma unroll
      for (int tm = 0; tm < 2; tm++) {
        mma16816<kDt>(acc[tm][2 * tp], a[tm], b[0], b[1]);
        mma16816<kDt>(acc[tm][2 * tp + 1], a[tm], b[2], b[3]);
      }
    }
  }
}

__device__ __forceinline__ void zero_acc(float (&acc)[2][8][4]) {
#pragma unroll
  for (int tm = 0; tm < 2; tm++)
#pragma unroll
    for (int tn = 0; tn < 8; tn++)
#pragma unroll
      for (int e = 0; e < 4; e++) acc[tm][tn][e] = 0.f;
}

// Two floats as a 16-bit pair of the element type (the lower first).
template <int kDt>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  return kDt == 1 ? pack_f16x2(lo, hi) : pack_bf16x2(lo, hi);
}

template <int kDt>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_kernel(const BwdParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint16_t* sQ = reinterpret_cast<uint16_t*>(smem_raw);
  uint16_t* sG = sQ + kTileElems;  // dO
  uint16_t* sK = sG + kTileElems;
  uint16_t* sV = sK + kTileElems;
  uint16_t* sP = sV + kTileElems;   // P [row][key], in the element type
  uint16_t* sS = sP + kTileElems;   // dS [row][key]
  float* sL = reinterpret_cast<float*>(sS + kTileElems);  // lse * log2(e), -inf: no weight
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

  // rows of this tile: token offset r / G in the tile, head r % G (a token
  // past T, which only inconsistent lengths give, is left alone: the
  // metadata status has flagged them)
  auto row_tok = [&](int r) { return s * p.tile_tokens + r / p.G; };
  auto in_t = [&](int r) { return tok_begin + row_tok(r) < p.T; };
  auto row_valid = [&](int r) { return r < rows_in_tile && row_tok(r) < n_store && in_t(r); };
  auto row_used = [&](int r) { return r < rows_in_tile && row_tok(r) < n_used && in_t(r); };
  auto row_index = [&](int r) {  // (token, head) row of q / dq
    return ((int64_t)(tok_begin + row_tok(r)) * p.N1 + kvh * p.G + r % p.G);
  };
  load_tiles(sQ, sG, [&](int r) { return row_used(r) ? p.q + row_index(r) * kHeadDim : nullptr; },
             [&](int r) { return row_used(r) ? p.dout + row_index(r) * kHeadDim : nullptr; });
  if (threadIdx.x < 128) {
    const int r = threadIdx.x;
    const bool used = row_used(r);
    const float l = used ? p.lse[row_index(r)] : -INFINITY;
    sL[r] = l * 1.4426950408889634f;
    sD[r] = used ? p.delta[row_index(r)] : 0.f;
    sPos[r] = pos0 + row_tok(r);
  }

  // warp w owns rows (or keys) 32 (w >> 1) .. + 31 and columns 64 (w & 1) .. + 63
  // of every 128 x 128 product; a fragment element e of tile (tm, tn) sits at
  // row m0 + 16 tm + lane / 4 + 8 (e >> 1), column n0 + 8 tn + 2 (lane % 4) + (e & 1)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = 32 * (warp >> 1), n0 = 64 * (warp & 1);
  const int fr = lane >> 2, fc = 2 * (lane & 3);
  float dq[2][8][4];
  zero_acc(dq);

  const int32_t* list = meta + off_list + (int64_t)item * p.top_k;
  const bool tnd = p.cu_kv != nullptr;
  int32_t bad = 0;
  // block e of the list: its first row in k / v (rows of N2 * D elements; a
  // page is kv_page_stride elements) and in the compact dk / dv; ok = false
  // for a page index out of range (the block then gets no weight)
  struct Blk {
    int32_t lb;
    int64_t row0, grow0;
    bool ok;
  };
  const int64_t page_rows = tnd ? 0 : p.kv_page_stride / ((int64_t)p.N2 * kHeadDim);
  auto block_of = [&](int32_t e) {
    Blk x;
    x.lb = list[e] & kEntryLbMask;
    x.ok = true;
    if (tnd) {
      x.row0 = x.grow0 = p.cu_kv[b] + (int64_t)x.lb * kPage;
    } else {
      const int32_t page =
          x.lb < p.max_pages ? p.block_table[(int64_t)b * p.max_pages + x.lb] : -1;
      x.ok = page >= 0 && page < p.num_pages;
      x.row0 = x.ok ? (int64_t)page * page_rows : 0;
      x.grow0 = x.ok ? (int64_t)page * kPage : 0;
    }
    return x;
  };
  auto key_ok = [&](const Blk& x, int c) {
    const int64_t key = (int64_t)x.lb * kPage + c;
    return x.ok && key < ku && (!tnd || x.row0 + c < p.T_kv);
  };
  // asynchronous copy of block x's K or V tile (rows past seqused_kv, and a
  // block with no weight, are zero-filled)
  auto fetch = [&](uint16_t* tile, const uint16_t* src, const Blk& x) {
#pragma unroll
    for (int it = 0; it < kChunksPerThread; it++) {
      const int i = threadIdx.x + it * kBwdThreads;
      const int r = i >> 4, c = i & 15;
      const bool ok = key_ok(x, r);
      cp_async16(tile + r * kRowElems + 8 * c,
                 ok ? src + ((x.row0 + r) * p.N2 + kvh) * kHeadDim + 8 * c : src, ok ? 16u : 0u);
    }
  };
  if (n_live > 0) {
    const Blk x0 = block_of(0);
    fetch(sK, p.k, x0);
    fetch(sV, p.v, x0);
    cp_async_commit();
  }
  for (int32_t e = 0; e < n_live; e++) {
    // K and V of block e were fetched during block e - 1 (or above); the
    // next block's are fetched as soon as each tile is free: V after dP,
    // K after dQ
    const Blk x = block_of(e);
    if (!x.ok) bad |= kDevBadPage;
    const int32_t lb = x.lb;
    const bool has_next = e + 1 < n_live;
    const Blk xn = block_of(has_next ? e + 1 : e);
    cp_async_wait_all();
    __syncthreads();

    float acc[2][8][4];
    // ---- S = Q K^T, then P = exp(s - lse) on visible (row, key) pairs
    zero_acc(acc);
    warp_gemm<kDt, false, false>(acc, sQ, sK, m0, n0);
#pragma unroll
    for (int tm = 0; tm < 2; tm++)
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int r = m0 + 16 * tm + fr + 8 * h;
        const int32_t pos = sPos[r];
        const float l2 = sL[r];
#pragma unroll
        for (int tn = 0; tn < 8; tn++) {
          const int c = n0 + 8 * tn + fc;
          float pv[2];
#pragma unroll
          for (int u = 0; u < 2; u++) {
            const int32_t key = lb * kPage + c + u;
            const bool vis = x.ok && l2 != -INFINITY && key < ku && key <= pos &&
                             (p.win_left < 0 || key >= pos - p.win_left);
            pv[u] = vis ? fast_exp2(acc[tm][tn][2 * h + u] * p.scale_log2 - l2) : 0.f;
          }
          *reinterpret_cast<uint32_t*>(sP + r * kRowElems + c) = pack2<kDt>(pv[0], pv[1]);
        }
      }
    __syncthreads();

    // ---- dV = P^T dO   (rows: keys, columns: head dim)
    zero_acc(acc);
    warp_gemm<kDt, true, true>(acc, sP, sG, m0, n0);
#pragma unroll
    for (int tm = 0; tm < 2; tm++)
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int c = m0 + 16 * tm + fr + 8 * h;
        if (!key_ok(x, c)) continue;
        float2* dst = reinterpret_cast<float2*>(p.dv + ((x.grow0 + c) * p.N2 + kvh) * kHeadDim);
#pragma unroll
        for (int tn = 0; tn < 8; tn++)
          atomicAdd(dst + ((n0 + 8 * tn + fc) >> 1),
                    make_float2(acc[tm][tn][2 * h], acc[tm][tn][2 * h + 1]));
      }

    // ---- dS = P (dO V^T - delta)   (P as the products use it: 16-bit)
    zero_acc(acc);
    warp_gemm<kDt, false, false>(acc, sG, sV, m0, n0);
#pragma unroll
    for (int tm = 0; tm < 2; tm++)
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int r = m0 + 16 * tm + fr + 8 * h;
        const float dlt = sD[r];
#pragma unroll
        for (int tn = 0; tn < 8; tn++) {
          const int c = n0 + 8 * tn + fc;
          const float2 pv = widen2<kDt>(*reinterpret_cast<const uint32_t*>(sP + r * kRowElems + c));
          *reinterpret_cast<uint32_t*>(sS + r * kRowElems + c) =
              pack2<kDt>(pv.x * (acc[tm][tn][2 * h] - dlt), pv.y * (acc[tm][tn][2 * h + 1] - dlt));
        }
      }
    __syncthreads();  // dS is complete and V no longer read
    if (has_next) {
      fetch(sV, p.v, xn);
      cp_async_commit();
    }

    // ---- dQ += dS K   (rows: queries, columns: head dim)
    warp_gemm<kDt, false, true>(dq, sS, sK, m0, n0);
    __syncthreads();  // K no longer read
    if (has_next) {
      fetch(sK, p.k, xn);
      cp_async_commit();
    }

    // ---- dK = scale dS^T Q   (rows: keys, columns: head dim)
    zero_acc(acc);
    warp_gemm<kDt, true, true>(acc, sS, sQ, m0, n0);
#pragma unroll
    for (int tm = 0; tm < 2; tm++)
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int c = m0 + 16 * tm + fr + 8 * h;
        if (!key_ok(x, c)) continue;
        float2* dst = reinterpret_cast<float2*>(p.dk + ((x.grow0 + c) * p.N2 + kvh) * kHeadDim);
#pragma unroll
        for (int tn = 0; tn < 8; tn++)
          atomicAdd(dst + ((n0 + 8 * tn + fc) >> 1),
                    make_float2(acc[tm][tn][2 * h] * p.scale, acc[tm][tn][2 * h + 1] * p.scale));
      }
  }

  // dQ of the tile's stored rows (0 for rows past seqused_q or with no key)
#pragma unroll
  for (int tm = 0; tm < 2; tm++)
#pragma unroll
    for (int h = 0; h < 2; h++) {
      const int r = m0 + 16 * tm + fr + 8 * h;
      if (!row_valid(r)) continue;
      float2* dst = reinterpret_cast<float2*>(p.dq + row_index(r) * kHeadDim);
#pragma unroll
      for (int tn = 0; tn < 8; tn++)
        dst[(n0 + 8 * tn + fc) >> 1] =
            make_float2(dq[tm][tn][2 * h] * p.scale, dq[tm][tn][2 * h + 1] * p.scale);
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
