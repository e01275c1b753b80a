// gbsa_meta.cu -- metadata kernels: the deterministic, load-balanced work
// list of (Q block, KV head, tile pair, KV-block range) units, with split-KV
// pieces for long lists and the combine records that merge them.
//
// GBSA article (cf-1.com/news/4865651), "two-phase call": a metadata operator
// runs before the attention and records the task split that balances the
// load across cores; "Constraints": the metadata must match the operator's
// attributes, Q blocks are counted over storage lengths while the task space
// follows seqused, and values are not validated on the host (here the
// kernels record GBSA_DEV_* bits instead).
//
// Launches on the caller's stream:
//   1. seq_kernel   (1 CTA, only for more than 1024 sequences): per-sequence
//                   lengths, Q-block bases, header; with fewer sequences every
//                   item CTA derives them itself and CTA 0 writes them;
//   2. item_kernel  (1 warp per item): liveness of every list entry, the
//                   compacted live list with mask / partial-page flags;
//   3. plan_kernel  (1 CTA):  split length, pieces, longest-first order
//                   (a stable counting sort by piece length), split slots and
//                   combine records.
#include <cuda_runtime.h>
#include <stdint.h>

#include "gbsa.h"
#include "gbsa_internal.cuh"

namespace gbsa {

namespace {

constexpr int kSeqThreads = 1024;
constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;
constexpr int kNumKeys = kMaxTopK + 1;  // piece lengths 0..256

__device__ __forceinline__ int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }

__device__ __forceinline__ void raise_status(const MetaParams& p, int32_t bits) {
  if (bits) {
    atomicOr(&p.meta[H_STATUS], bits);
    if (p.dev_status) atomicOr(p.dev_status, bits);
  }
}

// Block-wide exclusive scan of one int64 per thread (blockDim.x threads,
// a multiple of 32, at most 1024).  `scratch` holds 33 int64: the warps'
// prefixes and, apart from them, the block sum.  Returns the exclusive
// prefix; *total gets the block sum.
__device__ int64_t block_exclusive_scan(int64_t v, int64_t* scratch, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int64_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  __syncthreads();
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < nwarps ? scratch[lane] : 0;
    int64_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    if (lane < nwarps) scratch[lane] = wi - w;
    if (lane == 31) scratch[32] = wi;  // lanes >= nwarps add 0, so lane 31 holds the sum
  }
  __syncthreads();
  const int64_t res = scratch[warp] + incl - v;
  *total = scratch[32];
  __syncthreads();
  return res;
}

// ---------------------------------------------------------------------------
// 1. sequences
// ---------------------------------------------------------------------------
// Header fields known before the plan, the sequence status, and the (at most
// 3) padding words between the live lists and the unit table.
__device__ void write_header(const MetaParams& p, int32_t status) {
  const Geometry& g = p.geo;
  int32_t* meta = p.meta;
  meta[H_MAGIC] = (int32_t)kMagic;
  meta[H_VERSION] = kFormatVersion;
  meta[H_SIGNATURE] = (int32_t)p.signature;
  meta[H_B] = p.B;
  meta[H_NITEMS] = g.n_items;
  meta[H_TILE_TOKENS] = g.tile_tokens;
  meta[H_TILES_MAX] = g.tiles_max;
  meta[H_NUM_CTAS] = p.num_ctas;
  meta[H_UNIT_CAP] = (int32_t)g.unit_cap;
  meta[H_SLOT_CAP] = (int32_t)g.slot_cap;
  meta[H_COMB_CAP] = (int32_t)g.comb_cap;
  meta[H_STATUS] = status;
  meta[H_OFF_SEQ] = (int32_t)g.off_seq;
  meta[H_OFF_ITEM] = (int32_t)g.off_item;
  meta[H_OFF_LIST] = (int32_t)g.off_list;
  meta[H_OFF_UNIT] = (int32_t)g.off_unit;
  meta[H_OFF_COMB] = (int32_t)g.off_comb;
  meta[H_TOTAL] = (int32_t)g.total_words;
  meta[H_ROWS_PER_UNIT] = g.rows_per_unit;
  meta[H_G] = g.G;
  for (int64_t w = g.off_list + (int64_t)g.n_items * p.top_k; w < g.off_unit; w++) meta[w] = 0;
  if (status && p.dev_status) atomicOr(p.dev_status, status);
}

int32_t seq_threads(int32_t B) {
  const int32_t t = (B + 31) / 32 * 32;
  return t < kSeqThreads ? t : kSeqThreads;
}

__global__ void __launch_bounds__(kSeqThreads) seq_kernel(const MetaParams p) {
  __shared__ int64_t scratch[33];
  __shared__ int64_t ends_sh[2];  // cu_seqlens_q[0], cu_seqlens_q[B]
  __shared__ int32_t bad_sh;
  const Geometry& g = p.geo;
  int32_t* meta = p.meta;
  allow_dependents();
  if (threadIdx.x == 0) {
    ends_sh[0] = p.cu_seqlens_q[0];
    ends_sh[1] = p.cu_seqlens_q[p.B];
    bad_sh = 0;
  }
  if (threadIdx.x < kHeaderWords) meta[threadIdx.x] = 0;
  __syncthreads();
  int32_t bad = 0;
  int64_t running = 0;
  for (int64_t base = 0; base < p.B; base += blockDim.x) {
    const int64_t b = base + threadIdx.x;
    int64_t nqb = 0, qs = 0, qu = 0, ku = 0, tok = 0;
    if (b < p.B) {
      tok = p.cu_seqlens_q[b];
      qs = p.cu_seqlens_q[b + 1] - tok;
      qu = p.has_seqused_q ? (int64_t)p.seqused_q[b] : qs;
      ku = p.seqused_kv[b];
      if (qs < 0 || qu < 0 || qu > qs || ku < 0) bad = 1;
      nqb = qs > 0 ? cdiv64(qs, p.block_x) : 0;
    }
    int64_t total;
    const int64_t excl = block_exclusive_scan(nqb, scratch, &total);
    if (b < p.B) {
      int4* row = reinterpret_cast<int4*>(meta + g.off_seq + 8 * b);
      row[0] = make_int4((int32_t)qs, (int32_t)qu, (int32_t)ku, (int32_t)nqb);
      row[1] = make_int4((int32_t)(running + excl), (int32_t)tok, 0, 0);
    }
    running += total;
  }
  if (bad) atomicOr(&bad_sh, 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    const int64_t c0 = ends_sh[0], cB = ends_sh[1];
    if (bad_sh || c0 != 0 || running != p.total_q_blocks || (p.T > 0 && cB != p.T) ||
        cB > 0x7fffffffLL)
      bad = kDevBadSeqlen;
    else
      bad = 0;
    write_header(p, bad);
  }
}

// ---------------------------------------------------------------------------
// 2. items: one warp per (Q block, KV head)
// ---------------------------------------------------------------------------
constexpr int kItemWarps = 8;
constexpr int kItemThreads = kItemWarps * 32;
constexpr int kItemSmemSeqs = 2048;  // sequences whose Q-block bases are staged
constexpr int kOwnSeqMax = GBSA_METADATA_FUSED_MAX_B;  // up to this many sequences,
                                     // every item CTA derives the sequence table itself
constexpr int kOwnSeqPer = kOwnSeqMax / kItemThreads;
static_assert(kOwnSeqMax % kItemThreads == 0, "whole sequences per item thread");
constexpr int kListChunks = kMaxTopK / 32;

// Status bits of item i go to word i of the unit table (rows there are
// undefined until the plan kernel writes them); the plan kernel ORs them
// into the header.  No word of the buffer has to be zeroed first.
__device__ __forceinline__ int32_t* item_status_word(const MetaParams& p, int64_t item) {
  return p.meta + p.geo.off_unit + item;
}

// kOwnSeq: the first kernel of the call; each CTA computes the per-sequence
// fields and Q-block bases of all B <= kOwnSeqMax sequences into shared
// memory, and CTA 0 writes the sequence table and the header.  Otherwise the
// sequence kernel ran before and the bases are read back from its table.
template <bool kOwnSeq>
__global__ void __launch_bounds__(kItemThreads) item_kernel(const MetaParams p) {
  constexpr int kCap = kOwnSeq ? kOwnSeqMax : kItemSmemSeqs;
  __shared__ int32_t base_sh[kCap];                    // first Q block of each sequence
  __shared__ int32_t nqb_sh[kCap];                     // its Q-block count
  __shared__ int4 row_sh[kOwnSeq ? kOwnSeqMax : 1];    // (qs, qu, ku, first token)
  __shared__ int64_t scratch[33];
  __shared__ int32_t bad_sh;
  allow_dependents();
  const Geometry& g = p.geo;
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * kItemWarps + (threadIdx.x >> 5);
  const bool active = item < g.n_items;
  const int32_t qb = (int32_t)(item / p.N2);
  const int32_t kvh = (int32_t)(item % p.N2);

  // The selection list and count are inputs of the call, complete before the
  // first kernel of the call started: read them before any wait.
  int64_t n = 0;
  int32_t pre[kListChunks];
  const int32_t* list = p.sparse_idx + ((int64_t)kvh * p.total_q_blocks + qb) * p.top_k;
  if (active) n = p.sparse_count[(int64_t)kvh * p.total_q_blocks + qb];
#pragma unroll
  for (int c = 0; c < kListChunks; c++) {
    const int32_t j = 32 * c + lane;
    pre[c] = (active && j < p.top_k) ? list[j] : 0;
  }

  const int32_t* seq = p.meta + g.off_seq;
  bool staged = true;
  if constexpr (kOwnSeq) {
    const int t = threadIdx.x;
    int64_t c0 = 0, cB = 0;  // the header's checks, loaded early
    if (blockIdx.x == 0 && t == 0) {
      c0 = p.cu_seqlens_q[0];
      cB = p.cu_seqlens_q[p.B];
    }
    if (t == 0) bad_sh = 0;
    int64_t nq[kOwnSeqPer];
    int64_t sum = 0;
    int32_t bad = 0;
#pragma unroll
    for (int r = 0; r < kOwnSeqPer; r++) {
      const int32_t b = kOwnSeqPer * t + r;
      nq[r] = 0;
      if (b < p.B) {
        const int64_t tok = p.cu_seqlens_q[b];
        const int64_t qs = p.cu_seqlens_q[b + 1] - tok;
        const int64_t qu = p.has_seqused_q ? (int64_t)p.seqused_q[b] : qs;
        const int64_t ku = p.seqused_kv[b];
        if (qs < 0 || qu < 0 || qu > qs || ku < 0) bad = 1;
        nq[r] = qs > 0 ? cdiv64(qs, p.block_x) : 0;
        row_sh[b] = make_int4((int32_t)qs, (int32_t)qu, (int32_t)ku, (int32_t)tok);
        nqb_sh[b] = (int32_t)nq[r];
      }
      sum += nq[r];
    }
    int64_t total;
    int64_t run = block_exclusive_scan(sum, scratch, &total);  // its barriers publish row_sh
#pragma unroll
    for (int r = 0; r < kOwnSeqPer; r++) {
      const int32_t b = kOwnSeqPer * t + r;
      if (b < p.B) base_sh[b] = (int32_t)run;
      run += nq[r];
    }
    if (bad) atomicOr(&bad_sh, 1);
    if (blockIdx.x == 0) {
      int32_t* meta = p.meta;
      if (t < kHeaderWords) meta[t] = 0;
#pragma unroll
      for (int r = 0; r < kOwnSeqPer; r++) {
        const int32_t b = kOwnSeqPer * t + r;
        if (b < p.B) {
          const int4 q = row_sh[b];
          int4* row = reinterpret_cast<int4*>(meta + g.off_seq + 8 * (int64_t)b);
          row[0] = make_int4(q.x, q.y, q.z, nqb_sh[b]);
          row[1] = make_int4(base_sh[b], q.w, 0, 0);
        }
      }
      __syncthreads();  // bad_sh complete; the zeroed header before its fields
      if (t == 0) {
        const int32_t st = (bad_sh || c0 != 0 || total != p.total_q_blocks ||
                            (p.T > 0 && cB != p.T) || cB > 0x7fffffffLL)
                               ? kDevBadSeqlen
                               : 0;
        write_header(p, st);
      }
    }
    __syncthreads();
  } else {
    grid_dependency_wait();  // the sequence table
    staged = p.B <= kItemSmemSeqs;
    if (staged) {
      for (int32_t b = threadIdx.x; b < p.B; b += kItemThreads) {
        nqb_sh[b] = seq[8 * b + 3];
        base_sh[b] = seq[8 * b + 4];
      }
    }
    __syncthreads();
  }
  if (!active) return;
  auto seq_base = [&](int32_t b) { return staged ? base_sh[b] : seq[8 * b + 4]; };
  auto seq_nqb = [&](int32_t b) { return staged ? nqb_sh[b] : seq[8 * b + 3]; };

  // sequence holding Q block qb: the last b with a block starting at or before qb
  int32_t lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (seq_base(mid) <= qb) lo = mid; else hi = mid - 1;
  }
  int32_t b = lo;
  while (b > 0 && seq_nqb(b) == 0) b--;
  int64_t qs, qu, ku, tok0;
  if constexpr (kOwnSeq) {
    const int4 r = row_sh[b];
    qs = r.x;
    qu = r.y;
    ku = r.z;
    tok0 = r.w;
  } else {
    const int4 r = *reinterpret_cast<const int4*>(seq + 8 * b);  // qs, qu, ku, nqb
    qs = r.x;
    qu = r.y;
    ku = r.z;
    tok0 = seq[8 * b + 5];
  }
  const int64_t qbl = (int64_t)qb - seq_base(b);
  const int64_t bx = p.block_x;
  int64_t n_store = qs - qbl * bx;
  if (n_store > bx) n_store = bx;
  if (n_store < 0) n_store = 0;
  int64_t n_used = qu - qbl * bx;
  if (n_used > n_store) n_used = n_store;
  if (n_used < 0) n_used = 0;
  const int64_t n_tiles = cdiv64(n_store, g.tile_tokens);
  const int64_t pos0 = qbl * bx + ku - qu;
  const int64_t p_hi = pos0 + n_used - 1;
  const int64_t nblk = cdiv64(ku, kPage);
  const int64_t wl = p.win_left;

  int32_t bits = 0;
  if (n < 0 || n > p.top_k) {
    bits |= kDevBadCount;
    n = n < 0 ? 0 : p.top_k;
  }
  int32_t* out_list = p.meta + g.off_list + item * p.top_k;
  int32_t n_live = 0;
#pragma unroll
  for (int c = 0; c < kListChunks; c++) {
    if (32 * c >= p.top_k) break;
    const int64_t j = 32 * c + lane;
    int32_t entry = 0;
    bool live = false;
    if (j < n) {
      const int64_t lb = pre[c];
      if (lb < 0 || lb >= nblk) {
        bits |= kDevBadBlockIdx;
      } else if (n_used > 0) {
        const int64_t k_lo = lb * kPage;
        const int64_t k_hi = (k_lo + kPage - 1 < ku - 1) ? k_lo + kPage - 1 : ku - 1;
        live = k_lo <= p_hi && (wl < 0 || k_hi + wl >= pos0);
        const bool full = k_lo + kPage <= ku && k_lo + kPage - 1 <= pos0 &&
                          (wl < 0 || k_lo >= p_hi - wl);
        entry = (int32_t)lb | (full ? 0 : kEntryMask) | (k_lo + kPage > ku ? kEntryPartial : 0);
      }
    }
    const uint32_t ballot = __ballot_sync(0xffffffffu, live);
    const int32_t before = __popc(ballot & ((1u << lane) - 1u));
    if (live) out_list[n_live + before] = entry;
    n_live += __popc(ballot);
  }
  for (int64_t j = n_live + lane; j < p.top_k; j += 32) out_list[j] = 0;
  bits = __reduce_or_sync(0xffffffffu, bits);
  if (lane == 0) {
    int4* row = reinterpret_cast<int4*>(p.meta + g.off_item + 8 * item);
    row[0] = make_int4(b, n_live, (int32_t)n_tiles, (int32_t)(tok0 + qbl * bx));
    row[1] = make_int4((int32_t)n_store, (int32_t)n_used, (int32_t)pos0, (int32_t)ku);
    *item_status_word(p, item) = bits;
    if (bits && p.dev_status) atomicOr(p.dev_status, bits);
  }
}

// ---------------------------------------------------------------------------
// 3. plan: split-KV pieces, longest-first order, slots and combine records
// ---------------------------------------------------------------------------
struct PieceShape {
  int32_t U;       // tile pairs of the item
  int32_t n;       // live blocks
  int32_t k;       // pieces per tile pair
  int32_t a;       // short piece length floor(n/k); long pieces have a+1
  int32_t cA, cB;  // long / short pieces per tile pair
};

__device__ __forceinline__ PieceShape piece_shape(int32_t U, int32_t n, int32_t L) {
  PieceShape s;
  s.U = U;
  s.n = n;
  if (n <= L) {
    s.k = 1;
    s.a = n;
    s.cA = 0;
    s.cB = 1;
  } else {
    s.k = (int32_t)(((uint32_t)n + (uint32_t)L - 1u) / (uint32_t)L);
    s.a = (int32_t)((uint32_t)n / (uint32_t)s.k);
    s.cA = n - s.k * s.a;
    s.cB = s.k - s.cA;
  }
  return s;
}

// Warp sum of non-negative int64 values, exact while each is below 2^30; a
// value at or above 2^30 makes the sum at least 2^30, past every capacity.
__device__ __forceinline__ int64_t warp_sum_sat(int64_t v) {
  const uint32_t c = v < (1LL << 30) ? (uint32_t)v : (1u << 30);
  const uint32_t lo = __reduce_add_sync(0xffffffffu, c & 0xffffu);
  const uint32_t hi = __reduce_add_sync(0xffffffffu, c >> 16);
  return ((int64_t)hi << 16) + lo;
}

// Item fields (tile pairs U, live blocks n) of the first kPlanSmemItems items
// are staged in dynamic shared memory; later items are re-read from the item
// table.
constexpr int kPlanSmemItems = 24576;
constexpr int kKeyBits = 9;          // piece lengths 0..256 (and 257 as a query)
constexpr int32_t kNoKey = 511;      // lanes past the warp's items
constexpr int kKeyWarps = (kNumKeys + 31) / 32;  // warps holding one length per thread
constexpr int kKeyRow = 36;                      // words per length in the (length, warp) table
static_assert(kPlanWarps == 32 && kKeyRow % 4 == 0 && kKeyRow >= kPlanWarps, "table rows");

size_t plan_smem_bytes(int64_t n_items) {
  const int64_t c = n_items < kPlanSmemItems ? n_items : kPlanSmemItems;
  return (size_t)(c * 6 + 16);
}

// The piece order is a stable counting sort of all pieces by length, longest
// first; inside a length, pieces follow their item, then tile pair, then
// their place in the item's split.  Warp w owns the contiguous item range
// [w R, (w + 1) R), R = ceil(items / 32) rounded up to a multiple of 32 (so
// small lists use fewer, fuller warps), and walks it 32 items at a time, so
// item order is (warp, step, lane) order:
//   pass 2  per (length, warp) piece counts, per-warp unit / slot / combine
//           totals;
//   scan    bucket starts (lengths descending), per-(length, warp) offsets
//           (warps ascending), per-warp slot and combine bases;
//   pass 3  each warp places its pieces with no block barrier: a piece's
//           rank inside its length is the warp's running cursor for that
//           length plus the weights of earlier lanes of the same step with
//           that length -- by match_any and a popcount when no lane splits
//           and all have equal tile pairs, else by pointer jumping over
//           lanes of equal keys.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const MetaParams p, int32_t cached) {
  extern __shared__ __align__(16) unsigned char plan_dyn[];
  __shared__ int64_t part[kPlanWarps][3];  // per warp: units, slots, combine records
  __shared__ int64_t totals[3];
  __shared__ int64_t key_warp_sum[kKeyWarps];
  __shared__ int32_t bucket_start[kNumKeys];
  // per (length, warp): counts, then running cursors.  A length's row is
  // 36 words: its 32 warps in 8 aligned int4, rows 16 B apart modulo 128 B
  // so that 8 lanes of a vector access reach 8 different bank groups.
  __shared__ __align__(16) int32_t key_warp[kNumKeys][kKeyRow];
  __shared__ int32_t split_len_sh;
  __shared__ int64_t cost_sh[kPlanWarps];
  __shared__ int32_t status_sh, item_bits_sh;
  int32_t* sU = reinterpret_cast<int32_t*>(plan_dyn);
  uint16_t* sN = reinterpret_cast<uint16_t*>(sU + cached);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kNumKeys * kKeyRow; i += blockDim.x) (&key_warp[0][0])[i] = 0;
  allow_dependents();
  grid_dependency_wait();  // the item table and live lists
  const Geometry& g = p.geo;
  int32_t* meta = p.meta;
  const int32_t* items = meta + g.off_item;
  const int32_t n_items = g.n_items;

  auto fields = [&](int32_t i, int32_t& U, int32_t& n) {
    if (i < cached) {
      U = sU[i];
      n = sN[i];
    } else {
      const int4 r = *reinterpret_cast<const int4*>(items + 8 * (int64_t)i);
      n = r.y;
      U = (r.z + 1) / 2;
    }
  };

  // stage the fields, total cost; the items' status bits (left in the unit
  // table's first words) go into the header
  if (tid == 0) {
    status_sh = meta[H_STATUS];
    item_bits_sh = 0;
  }
  int64_t cost = 0;
  int32_t ibits = 0;
  const int32_t* item_bits = meta + g.off_unit;
#pragma unroll 4
  for (int32_t i = tid; i < n_items; i += kPlanThreads) {
    // item rows are 8 words on a 16-byte boundary: (.., n, n_tiles, ..)
    const int4 r = *reinterpret_cast<const int4*>(items + 8 * (int64_t)i);
    ibits |= item_bits[i];
    const int32_t U = (r.z + 1) / 2;
    if (i < cached) {
      sU[i] = U;
      sN[i] = (uint16_t)r.y;
    }
    cost += (int64_t)U * r.y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cost += __shfl_xor_sync(0xffffffffu, cost, o);
  ibits = __reduce_or_sync(0xffffffffu, ibits);
  if (lane == 0) {
    cost_sh[warp] = cost;
    if (ibits) atomicOr(&item_bits_sh, ibits);
  }
  __syncthreads();
  if (tid == 0) meta[H_STATUS] = status_sh | item_bits_sh;
  if (status_sh & kDevBadSeqlen) {
    if (tid == 0) {
      meta[H_NUNITS] = 0;
      meta[H_NSLOTS] = 0;
      meta[H_NCOMB] = 0;
      meta[H_SPLIT_LEN] = 0;
      meta[H_COST_LO] = 0;
      meta[H_COST_HI] = 0;
    }
    return;
  }
  // the split length, once (warp 0)
  if (warp == 0) {
    cost = cost_sh[lane];  // kPlanWarps == 32: one warp total per lane
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cost += __shfl_xor_sync(0xffffffffu, cost, o);
    if (lane == 0) {
      int64_t L64;
      if (p.forced_split > 0) {
        L64 = p.forced_split;
      } else {
        const int64_t d = 4LL * p.num_ctas;
        if (cost <= 0xffffffffLL && d <= 0xffffffffLL) {  // a 32-bit division
          const uint32_t q = (uint32_t)cost / (uint32_t)d;
          L64 = (int64_t)q + ((uint32_t)cost - q * (uint32_t)d != 0u ? 1 : 0);
        } else {
          L64 = cdiv64(cost, d);
        }
        if (L64 < kMinSplitLen) L64 = kMinSplitLen;
      }
      if (L64 > 0x7fffffffLL) L64 = 0x7fffffffLL;
      split_len_sh = (int32_t)L64;
      meta[H_SPLIT_LEN] = (int32_t)L64;
      meta[H_COST_LO] = (int32_t)(uint32_t)(cost & 0xffffffffLL);
      meta[H_COST_HI] = (int32_t)(uint32_t)((uint64_t)cost >> 32);
    }
  }
  __syncthreads();
  const int32_t L = split_len_sh;

  // each warp's range is a whole number of 32-item steps: fewer, fuller warps
  const int32_t R = ((n_items + kPlanWarps - 1) / kPlanWarps + 31) / 32 * 32;
  const int32_t lo = warp * R < n_items ? warp * R : n_items;
  const int32_t hi = lo + R < n_items ? lo + R : n_items;

  // pass 2: per (warp, length) counts and per-warp totals
  if (lo >= hi) {
    if (lane == 0) part[warp][0] = part[warp][1] = part[warp][2] = 0;
  } else {
    int64_t units = 0, slots = 0, combs = 0;
    for (int32_t i = lo + lane; i < hi; i += 32) {
      int32_t U, n;
      fields(i, U, n);
      const PieceShape s = piece_shape(U, n, L);
      atomicAdd(&key_warp[s.a][warp], s.U * s.cB);  // cB >= 1
      if (s.cA) atomicAdd(&key_warp[s.a + 1][warp], s.U * s.cA);
      units += (int64_t)s.U * s.k;
      if (s.k > 1) {
        slots += (int64_t)s.U * s.k;
        combs += s.U;
      }
    }
    const int64_t u = warp_sum_sat(units);
    const int64_t sl = __any_sync(0xffffffffu, slots != 0) ? warp_sum_sat(slots) : 0;
    const int64_t cb = sl ? warp_sum_sat(combs) : 0;
    if (lane == 0) {
      part[warp][0] = u;
      part[warp][1] = sl;
      part[warp][2] = cb;
    }
  }
  __syncthreads();

  // per length: offsets over warps, in place, and the length's total; thread
  // t < 257 takes length 256 - t, so the bucket starts (longest first) are an
  // exclusive scan over threads: inside each of the 9 warps here, across them
  // after the barrier.  The last warp scans the per-warp slot and combine
  // counts.
  int64_t key_excl = 0;
  if (tid < kKeyWarps * 32) {
    int32_t acc = 0;
    if (tid < kNumKeys) {
      const int key = kNumKeys - 1 - tid;
      // the length's 32 warp counts (idle warps' are zero) in 8 vector loads
      int4* row = reinterpret_cast<int4*>(&key_warp[key][0]);
      int4 c[kPlanWarps / 4];
#pragma unroll
      for (int v = 0; v < kPlanWarps / 4; v++) c[v] = row[v];
#pragma unroll
      for (int v = 0; v < kPlanWarps / 4; v++) {
        const int4 x = c[v];
        int4 e;
        e.x = acc;
        e.y = acc + x.x;
        e.z = e.y + x.y;
        e.w = e.z + x.z;
        acc = e.w + x.w;
        row[v] = e;
      }
    }
    int64_t incl = acc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    key_excl = incl - acc;
    if (lane == 31) key_warp_sum[warp] = incl;
  }
  if (warp == kPlanWarps - 1) {
    const int64_t u = part[lane][0], sl = part[lane][1], cb = part[lane][2];
    int64_t iu = u, is = sl, ic = cb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t nu = __shfl_up_sync(0xffffffffu, iu, o);
      const int64_t ns = __shfl_up_sync(0xffffffffu, is, o);
      const int64_t nc = __shfl_up_sync(0xffffffffu, ic, o);
      if (lane >= o) {
        iu += nu;
        is += ns;
        ic += nc;
      }
    }
    __syncwarp();
    part[lane][1] = is - sl;
    part[lane][2] = ic - cb;
    if (lane == 31) {
      totals[0] = iu;
      totals[1] = is;
      totals[2] = ic;
    }
  }
  __syncthreads();
  if (tid < kNumKeys) {
#pragma unroll
    for (int w = 0; w < kKeyWarps - 1; w++)
      if (w < warp) key_excl += key_warp_sum[w];
    bucket_start[kNumKeys - 1 - tid] = (int32_t)key_excl;
  }
  if (tid == 0) {
    const int64_t n_units = totals[0], n_slots = totals[1], n_comb = totals[2];
    const bool over = n_units > g.unit_cap || n_slots > g.slot_cap || n_comb > g.comb_cap;
    meta[H_NUNITS] = over ? 0 : (int32_t)n_units;
    meta[H_NSLOTS] = over ? 0 : (int32_t)n_slots;
    meta[H_NCOMB] = over ? 0 : (int32_t)n_comb;
    if (over) raise_status(p, kDevCapacity);
  }
  __syncthreads();
  if (totals[0] > g.unit_cap || totals[1] > g.slot_cap || totals[2] > g.comb_cap) return;

  // pass 3: place the pieces, warp by warp
  int4* units = reinterpret_cast<int4*>(meta + g.off_unit);
  int4* comb = reinterpret_cast<int4*>(meta + g.off_comb);
  int32_t slot_cur = (int32_t)part[warp][1], comb_cur = (int32_t)part[warp][2];
  const uint32_t lt = (1u << lane) - 1u, gt = ~lt & ~(1u << lane);
  for (int32_t base = lo; base < hi; base += 32) {
    const int32_t i = base + lane;
    const bool valid = i < hi;
    PieceShape s{0, 0, 1, 0, 0, 0};
    if (valid) {
      int32_t U, n;
      fields(i, U, n);
      s = piece_shape(U, n, L);
    }
    const int32_t a = valid ? s.a : kNoKey;
    const int32_t U0 = __shfl_sync(0xffffffffu, s.U, 0);  // lane 0 is always valid
    if (__all_sync(0xffffffffu, !valid || (s.k == 1 && s.U == U0))) {
      // no split and equal tile pairs: one piece of length n per tile pair,
      // rank = U0 x (earlier lanes with the same n)
      const uint32_t same = __match_any_sync(0xffffffffu, a);
      int32_t start = 0;
      if (valid) start = bucket_start[a] + key_warp[a][warp] + U0 * __popc(same & lt);
      __syncwarp();
      if (valid && !(same & gt)) key_warp[a][warp] += U0 * __popc(same);
      __syncwarp();
      if (valid)
        for (int32_t tp = 0; tp < U0; tp++) units[start + tp] = make_int4(i, tp, s.n << 16, -1);
      continue;
    }
    const int32_t wA = s.U * s.cA, wB = s.U * s.cB;  // 0 for lanes past the range
    // key-equality masks from the bits of a: eq(x) = lanes whose a == x
    uint32_t bal[kKeyBits];
#pragma unroll
    for (int b = 0; b < kKeyBits; b++) bal[b] = __ballot_sync(0xffffffffu, (a >> b) & 1);
    auto eq = [&](int32_t x) {
      uint32_t m = 0xffffffffu;
#pragma unroll
      for (int b = 0; b < kKeyBits; b++) m &= ((x >> b) & 1) ? bal[b] : ~bal[b];
      return m;
    };
    const uint32_t same = eq(a);
    // inclusive sums of wA and wB over the lanes <= this one with the same a
    int32_t sA = wA, sB = wB;
    int32_t ptr = (same & lt) ? 31 - __clz(same & lt) : -1;
    while (__any_sync(0xffffffffu, ptr >= 0)) {
      const int32_t src = ptr >= 0 ? ptr : lane;
      const int32_t tA = __shfl_sync(0xffffffffu, sA, src);
      const int32_t tB = __shfl_sync(0xffffffffu, sB, src);
      const int32_t tp = __shfl_sync(0xffffffffu, ptr, src);
      if (ptr >= 0) {
        sA += tA;
        sB += tB;
        ptr = tp;
      }
    }
    // length a gets the short pieces of lanes with a and the long pieces of
    // lanes with a - 1; length a + 1 the long pieces of lanes with a and the
    // short pieces of lanes with a + 1
    const uint32_t prev = (valid && a > 0) ? eq(a - 1) & lt : 0u;
    const uint32_t next = valid ? eq(a + 1) & lt : 0u;
    const int32_t xA = __shfl_sync(0xffffffffu, sA, prev ? 31 - __clz(prev) : lane);
    const int32_t xB = __shfl_sync(0xffffffffu, sB, next ? 31 - __clz(next) : lane);
    const int32_t preB = sB - wB + (prev ? xA : 0);
    const int32_t preA = sA - wA + (next ? xB : 0);
    // slots and combine records in item order (only split items have any)
    int32_t slot_base = 0, comb_base = 0;
    if (__any_sync(0xffffffffu, s.k > 1)) {
      const int32_t my_slots = s.k > 1 ? s.U * s.k : 0, my_combs = s.k > 1 ? s.U : 0;
      int32_t iS = my_slots, iC = my_combs;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t ns = __shfl_up_sync(0xffffffffu, iS, o);
        const int32_t nc = __shfl_up_sync(0xffffffffu, iC, o);
        if (lane >= o) {
          iS += ns;
          iC += nc;
        }
      }
      slot_base = slot_cur + iS - my_slots;
      comb_base = comb_cur + iC - my_combs;
      slot_cur += __shfl_sync(0xffffffffu, iS, 31);
      comb_cur += __shfl_sync(0xffffffffu, iC, 31);
    }
    int32_t startA = 0, startB = 0;
    if (valid) {
      startB = bucket_start[a] + key_warp[a][warp] + preB;
      if (s.cA) startA = bucket_start[a + 1] + key_warp[a + 1][warp] + preA;
    }
    __syncwarp();
    // the last lane of each key group advances the warp's cursors
    if (valid && !(same & gt)) {
      atomicAdd(&key_warp[a][warp], sB);
      if (sA) atomicAdd(&key_warp[a + 1][warp], sA);
    }
    __syncwarp();
    if (valid) {
      if (s.k > 1)
        for (int32_t tp = 0; tp < s.U; tp++)
          comb[comb_base + tp] = make_int4(i, tp, slot_base + tp * s.k, s.k);
      // piece q covers [floor(q n / k), floor((q + 1) n / k)); with n = a k + cA
      // the bound advances by a, plus 1 when (q + 1) cA mod k wraps: the
      // long pieces
      int32_t j0 = 0, longs = 0, rem = 0;
      for (int32_t q = 0; q < s.k; q++) {
        rem += s.cA;
        const bool is_long = rem >= s.k;
        if (is_long) rem -= s.k;
        const int32_t j1 = j0 + s.a + (is_long ? 1 : 0);
        const int32_t first = is_long ? startA + longs : startB + (q - longs);
        const int32_t stride = is_long ? s.cA : s.cB;
        for (int32_t tp = 0; tp < s.U; tp++)
          units[first + tp * stride] =
              make_int4(i, tp, j0 | (j1 << 16), s.k > 1 ? slot_base + tp * s.k + q : -1);
        longs += is_long ? 1 : 0;
        j0 = j1;
      }
    }
  }
}

}  // namespace

// Up to kOwnSeqMax sequences: two launches (items with their own sequence
// phase, then the plan); more: the sequence kernel first.  The later kernels
// start early (programmatic dependent launch) and wait for their inputs.
cudaError_t launch_metadata(const MetaParams& p, cudaStream_t stream) {
  const int64_t blocks = (p.geo.n_items + kItemWarps - 1) / kItemWarps;
  cudaError_t e;
  if (p.B <= kOwnSeqMax) {
    item_kernel<true><<<(unsigned)blocks, kItemThreads, 0, stream>>>(p);
    e = cudaGetLastError();
  } else {
    seq_kernel<<<1, seq_threads(p.B), 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_dependent(item_kernel<false>, dim3((unsigned)blocks), dim3(kItemThreads), 0,
                         stream, p);
  }
  if (e != cudaSuccess) return e;
  const int32_t cached = p.geo.n_items < kPlanSmemItems ? p.geo.n_items : kPlanSmemItems;
  const size_t smem = plan_smem_bytes(p.geo.n_items);
  if (smem > 8192) {
    e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_dependent(plan_kernel, dim3(1), dim3(kPlanThreads), smem, stream, p, cached);
}

}  // namespace gbsa
