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
// Three launches on the caller's stream:
//   1. seq_kernel   (1 CTA):  per-sequence lengths, Q-block bases, header;
//   2. item_kernel  (1 warp per item): liveness of every list entry, the
//                   compacted live list with mask / partial-page flags;
//   3. plan_kernel  (1 CTA):  split length, pieces, longest-first order
//                   (a stable counting sort by piece length), split slots and
//                   combine records.
#include <cuda_runtime.h>
#include <stdint.h>

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
// a multiple of 32, at most 1024).  `scratch` holds 32 int64.  Returns the
// exclusive prefix; *total gets the block sum.
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
    if (lane == 31) scratch[31] = wi;  // lanes >= nwarps add 0, so lane 31 holds the sum
  }
  __syncthreads();
  const int64_t res = scratch[warp] + incl - v;
  *total = scratch[31];
  __syncthreads();
  return res;
}

// ---------------------------------------------------------------------------
// 1. sequences
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kSeqThreads) seq_kernel(const MetaParams p) {
  __shared__ int64_t scratch[32];
  __shared__ int32_t bad_sh;
  const Geometry& g = p.geo;
  int32_t* meta = p.meta;
  allow_dependents();
  if (threadIdx.x == 0) bad_sh = 0;
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
      int32_t* row = meta + g.off_seq + 8 * b;
      row[0] = (int32_t)qs;
      row[1] = (int32_t)qu;
      row[2] = (int32_t)ku;
      row[3] = (int32_t)nqb;
      row[4] = (int32_t)(running + excl);
      row[5] = (int32_t)tok;
      row[6] = 0;
      row[7] = 0;
    }
    running += total;
  }
  if (bad) atomicOr(&bad_sh, 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    const int64_t c0 = p.cu_seqlens_q[0], cB = p.cu_seqlens_q[p.B];
    if (bad_sh || c0 != 0 || running != p.total_q_blocks || (p.T > 0 && cB != p.T) ||
        cB > 0x7fffffffLL)
      bad = kDevBadSeqlen;
    else
      bad = 0;
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
    meta[H_STATUS] = bad;
    meta[H_OFF_SEQ] = (int32_t)g.off_seq;
    meta[H_OFF_ITEM] = (int32_t)g.off_item;
    meta[H_OFF_LIST] = (int32_t)g.off_list;
    meta[H_OFF_UNIT] = (int32_t)g.off_unit;
    meta[H_OFF_COMB] = (int32_t)g.off_comb;
    meta[H_TOTAL] = (int32_t)g.total_words;
    meta[H_ROWS_PER_UNIT] = g.rows_per_unit;
    meta[H_G] = g.G;
    // the (at most 3) padding words between the live lists and the unit table
    for (int64_t w = g.off_list + (int64_t)g.n_items * p.top_k; w < g.off_unit; w++) meta[w] = 0;
    if (bad && p.dev_status) atomicOr(p.dev_status, bad);
  }
}

// ---------------------------------------------------------------------------
// 2. items: one warp per (Q block, KV head)
// ---------------------------------------------------------------------------
constexpr int kItemWarps = 8;

__global__ void __launch_bounds__(kItemWarps * 32) item_kernel(const MetaParams p) {
  allow_dependents();
  grid_dependency_wait();  // the sequence table
  const Geometry& g = p.geo;
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * kItemWarps + (threadIdx.x >> 5);
  if (item >= g.n_items) return;
  const int32_t* meta_c = p.meta;
  const int32_t qb = (int32_t)(item / p.N2);
  const int32_t kvh = (int32_t)(item % p.N2);
  const int32_t* seq = meta_c + g.off_seq;

  // sequence holding Q block qb: the last b with a block starting at or before qb
  int32_t lo = 0, hi = p.B - 1;
  while (lo < hi) {
    const int32_t mid = (lo + hi + 1) >> 1;
    if (seq[8 * mid + 4] <= qb) lo = mid; else hi = mid - 1;
  }
  int32_t b = lo;
  while (b > 0 && seq[8 * b + 3] == 0) b--;
  const int64_t qs = seq[8 * b + 0], qu = seq[8 * b + 1], ku = seq[8 * b + 2];
  const int64_t qbl = (int64_t)qb - seq[8 * b + 4];
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
  int64_t n = p.sparse_count[(int64_t)kvh * p.total_q_blocks + qb];
  if (n < 0 || n > p.top_k) {
    bits |= kDevBadCount;
    n = n < 0 ? 0 : p.top_k;
  }
  const int32_t* list = p.sparse_idx + ((int64_t)kvh * p.total_q_blocks + qb) * p.top_k;
  int32_t* out_list = p.meta + g.off_list + item * p.top_k;
  int32_t n_live = 0;
  for (int64_t j0 = 0; j0 < p.top_k; j0 += 32) {
    const int64_t j = j0 + lane;
    int32_t entry = 0;
    bool live = false;
    if (j < n) {
      const int64_t lb = list[j];
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
  if (lane == 0) {
    int32_t* row = p.meta + g.off_item + 8 * item;
    row[0] = b;
    row[1] = n_live;
    row[2] = (int32_t)n_tiles;
    row[3] = (int32_t)(seq[8 * b + 5] + qbl * bx);
    row[4] = (int32_t)n_store;
    row[5] = (int32_t)n_used;
    row[6] = (int32_t)pos0;
    row[7] = (int32_t)ku;
  }
  bits = __reduce_or_sync(0xffffffffu, bits);
  if (lane == 0) raise_status(p, bits);
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
  s.k = s.n <= L ? 1 : (s.n + L - 1) / L;
  s.a = s.n / s.k;
  s.cA = s.n - s.k * s.a;
  s.cB = s.k - s.cA;
  return s;
}

// Block-wide exclusive scans of NV int64 values per thread in one pass (one
// set of barriers).  `scratch` holds 32 * NV int64.  res[v] gets the
// exclusive prefix of v[v], total[v] the block sum.
template <int NV>
__device__ void block_exclusive_scan_n(const int64_t (&v)[NV], int64_t* scratch, int64_t (&res)[NV],
                                       int64_t (&total)[NV]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int64_t incl[NV];
#pragma unroll
  for (int c = 0; c < NV; c++) incl[c] = v[c];
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int c = 0; c < NV; c++) {
      const int64_t n = __shfl_up_sync(0xffffffffu, incl[c], o);
      if (lane >= o) incl[c] += n;
    }
  }
  __syncthreads();
  if (lane == 31) {
#pragma unroll
    for (int c = 0; c < NV; c++) scratch[32 * c + warp] = incl[c];
  }
  __syncthreads();
  if (warp < NV) {
    int64_t w = lane < nwarps ? scratch[32 * warp + lane] : 0;
    int64_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t n = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += n;
    }
    // lanes >= nwarps add 0, so lane 31's inclusive sum is the total; write
    // it after every lane has read its own slot
    __syncwarp();
    if (lane < nwarps) scratch[32 * warp + lane] = wi - w;
    if (lane == 31) scratch[32 * NV + warp] = wi;
  }
  __syncthreads();
#pragma unroll
  for (int c = 0; c < NV; c++) {
    res[c] = scratch[32 * c + warp] + incl[c] - v[c];
    total[c] = scratch[32 * NV + c];
  }
  __syncthreads();
}

// Item fields (tile pairs, live blocks) of the first kPlanCache chunks of
// blockDim items stay in registers across the three passes; further items
// are re-read from the item table.
constexpr int kPlanCache = 4;

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const MetaParams p) {
  __shared__ int64_t scratch[32 * 4];
  __shared__ int32_t hist[kNumKeys];
  __shared__ int32_t bucket_start[kNumKeys];
  __shared__ int32_t key_run[kNumKeys];
  __shared__ int32_t warp_key[kPlanWarps][kNumKeys];
  __shared__ int32_t split_len_sh;
  __shared__ int32_t abort_sh;

  allow_dependents();
  grid_dependency_wait();  // the item table and live lists
  const Geometry& g = p.geo;
  int32_t* meta = p.meta;
  const int32_t* items = meta + g.off_item;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t n_items = g.n_items;
  const int64_t chunks = (n_items + blockDim.x - 1) / blockDim.x;

  for (int i = tid; i < kNumKeys; i += blockDim.x) {
    hist[i] = 0;
    key_run[i] = 0;
  }
  for (int i = tid; i < kPlanWarps * kNumKeys; i += blockDim.x) (&warp_key[0][0])[i] = 0;
  if (tid == 0) abort_sh = (meta[H_STATUS] & kDevBadSeqlen) ? 1 : 0;

  // the item fields of this thread's items (chunk k: item k * blockDim + tid)
  int32_t cU[kPlanCache], cn[kPlanCache];
#pragma unroll
  for (int k = 0; k < kPlanCache; k++) {
    const int64_t i = (int64_t)k * blockDim.x + tid;
    cU[k] = 0;
    cn[k] = 0;
    if (i < n_items) {
      // item rows are 8 words on a 16-byte boundary: (.., n, n_tiles, ..)
      const int4 r = *reinterpret_cast<const int4*>(items + 8 * i);
      cn[k] = r.y;
      cU[k] = (r.z + 1) / 2;
    }
  }
  auto fields = [&](int64_t k, int32_t& U, int32_t& n) {
    U = 0;
    n = 0;
#pragma unroll
    for (int c = 0; c < kPlanCache; c++)
      if (c == k) {
        U = cU[c];
        n = cn[c];
      }
    if (k >= kPlanCache) {
      const int64_t i = k * blockDim.x + tid;
      if (i < n_items) {
        n = items[8 * i + 1];
        U = (items[8 * i + 2] + 1) / 2;
      }
    }
  };
  __syncthreads();
  if (abort_sh) {
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

  // pass 1: total cost
  int64_t cost = 0;
  for (int64_t k = 0; k < chunks; k++) {
    int32_t U, n;
    fields(k, U, n);
    cost += (int64_t)U * n;
  }
  {
    const int64_t v[1] = {cost};
    int64_t r[1], t[1];
    block_exclusive_scan_n<1>(v, scratch, r, t);
    cost = t[0];
  }
  if (tid == 0) {
    int64_t L;
    if (p.forced_split > 0) {
      L = p.forced_split;
    } else {
      L = cdiv64(cost, 4LL * p.num_ctas);
      if (L < kMinSplitLen) L = kMinSplitLen;
    }
    if (L > 0x7fffffffLL) L = 0x7fffffffLL;
    split_len_sh = (int32_t)L;
    meta[H_SPLIT_LEN] = (int32_t)L;
    meta[H_COST_LO] = (int32_t)(uint32_t)(cost & 0xffffffffLL);
    meta[H_COST_HI] = (int32_t)(uint32_t)((uint64_t)cost >> 32);
  }
  __syncthreads();
  const int32_t L = split_len_sh;

  // pass 2: histogram of piece lengths (weighted), totals
  int64_t pieces = 0, slots = 0, combs = 0;
  for (int64_t k = 0; k < chunks; k++) {
    int32_t U, n;
    fields(k, U, n);
    if (k * blockDim.x + tid >= n_items) continue;
    const PieceShape s = piece_shape(U, n, L);
    if (s.cA) atomicAdd(&hist[s.a + 1], s.U * s.cA);
    if (s.cB) atomicAdd(&hist[s.a], s.U * s.cB);
    pieces += (int64_t)s.U * s.k;
    if (s.k > 1) {
      slots += (int64_t)s.U * s.k;
      combs += s.U;
    }
  }
  int64_t n_units, n_slots, n_comb;
  {
    const int64_t v[3] = {pieces, slots, combs};
    int64_t r[3], t[3];
    block_exclusive_scan_n<3>(v, scratch, r, t);  // its barriers also publish hist
    n_units = t[0];
    n_slots = t[1];
    n_comb = t[2];
  }
  // bucket starts, longest first: an exclusive scan over the keys in
  // descending order (thread j holds key kNumKeys - 1 - j)
  {
    const int key = kNumKeys - 1 - tid;
    const int64_t v[1] = {tid < kNumKeys ? (int64_t)hist[key] : 0};
    int64_t r[1], t[1];
    block_exclusive_scan_n<1>(v, scratch, r, t);
    if (tid < kNumKeys) bucket_start[key] = (int32_t)r[0];
  }
  if (tid == 0) {
    const bool over = n_units > g.unit_cap || n_slots > g.slot_cap || n_comb > g.comb_cap;
    abort_sh = over ? 1 : 0;
    meta[H_NUNITS] = over ? 0 : (int32_t)n_units;
    meta[H_NSLOTS] = over ? 0 : (int32_t)n_slots;
    meta[H_NCOMB] = over ? 0 : (int32_t)n_comb;
    if (over) raise_status(p, kDevCapacity);
  }
  __syncthreads();
  if (abort_sh) return;

  // pass 3: place every piece (stable within a length), chunk by chunk
  int32_t* units = meta + g.off_unit;
  int32_t* comb = meta + g.off_comb;
  int64_t slot_run = 0, comb_run = 0;
  for (int64_t k = 0; k < chunks; k++) {
    const int64_t i = k * blockDim.x + tid;
    PieceShape s{0, 0, 1, 0, 0, 0};
    const bool valid = i < n_items;
    if (valid) {
      int32_t U, n;
      fields(k, U, n);
      s = piece_shape(U, n, L);
    }
    const int32_t kA = (valid && s.cA) ? s.a + 1 : -1;
    const int32_t wA = (valid && s.cA) ? s.U * s.cA : 0;
    const int32_t kB = (valid && s.cB) ? s.a : -1;
    const int32_t wB = (valid && s.cB) ? s.U * s.cB : 0;
    // per-key exclusive prefix inside the warp, in lane order
    int32_t preA = 0, preB = 0;
    for (int src = 0; src < 31; src++) {
      const int32_t ska = __shfl_sync(0xffffffffu, kA, src);
      const int32_t swa = __shfl_sync(0xffffffffu, wA, src);
      const int32_t skb = __shfl_sync(0xffffffffu, kB, src);
      const int32_t swb = __shfl_sync(0xffffffffu, wB, src);
      if (src < lane) {
        if (kA >= 0) preA += (ska == kA ? swa : 0) + (skb == kA ? swb : 0);
        if (kB >= 0) preB += (ska == kB ? swa : 0) + (skb == kB ? swb : 0);
      }
    }
    if (kA >= 0) atomicAdd(&warp_key[warp][kA], wA);
    if (kB >= 0) atomicAdd(&warp_key[warp][kB], wB);
    const int64_t my_slots = (valid && s.k > 1) ? (int64_t)s.U * s.k : 0;
    const int64_t my_combs = (valid && s.k > 1) ? s.U : 0;
    int64_t slot_base, comb_base;
    {
      const int64_t v[2] = {my_slots, my_combs};
      int64_t r[2], t[2];
      block_exclusive_scan_n<2>(v, scratch, r, t);  // its barriers also publish warp_key
      slot_base = slot_run + r[0];
      comb_base = comb_run + r[1];
      slot_run += t[0];
      comb_run += t[1];
    }
    // per key: exclusive prefix over warps, plus the run of earlier chunks
    for (int key = tid; key < kNumKeys; key += blockDim.x) {
      int32_t acc = key_run[key];
      for (int w = 0; w < kPlanWarps; w++) {
        const int32_t c = warp_key[w][key];
        warp_key[w][key] = acc;
        acc += c;
      }
      key_run[key] = acc;
    }
    __syncthreads();
    if (valid) {
      const int32_t startA = kA >= 0 ? bucket_start[kA] + warp_key[warp][kA] + preA : 0;
      const int32_t startB = kB >= 0 ? bucket_start[kB] + warp_key[warp][kB] + preB : 0;
      for (int32_t tp = 0; tp < s.U; tp++) {
        if (s.k > 1) {
          int32_t* c = comb + 4 * (comb_base + tp);
          c[0] = (int32_t)i;
          c[1] = tp;
          c[2] = (int32_t)(slot_base + (int64_t)tp * s.k);
          c[3] = s.k;
        }
        for (int32_t q = 0; q < s.k; q++) {
          const int32_t j0 = (int32_t)((int64_t)q * s.n / s.k);
          const int32_t j1 = (int32_t)((int64_t)(q + 1) * s.n / s.k);
          const int32_t longs_before = j0 - q * s.a;  // long pieces before q in this pair
          int32_t pos;
          if (j1 - j0 == s.a + 1 && s.cA)
            pos = startA + tp * s.cA + longs_before;
          else
            pos = startB + tp * s.cB + (q - longs_before);
          int32_t* u = units + 4 * (int64_t)pos;
          u[0] = (int32_t)i;
          u[1] = tp;
          u[2] = j0 | (j1 << 16);
          u[3] = s.k > 1 ? (int32_t)(slot_base + (int64_t)tp * s.k + q) : -1;
        }
      }
    }
    __syncthreads();
    for (int t = tid; t < kPlanWarps * kNumKeys; t += blockDim.x) (&warp_key[0][0])[t] = 0;
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_metadata(const MetaParams& p, cudaStream_t stream) {
  seq_kernel<<<1, kSeqThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t blocks = (p.geo.n_items + kItemWarps - 1) / kItemWarps;
  e = launch_dependent(item_kernel, dim3((unsigned)blocks), dim3(kItemWarps * 32), 0, stream, p);
  if (e != cudaSuccess) return e;
  return launch_dependent(plan_kernel, dim3(1), dim3(kPlanThreads), 0, stream, p);
}

}  // namespace gbsa
