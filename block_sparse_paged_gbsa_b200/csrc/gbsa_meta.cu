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
  s.k = s.n <= L ? 1 : (int32_t)(((uint32_t)s.n + (uint32_t)L - 1u) / (uint32_t)L);
  s.a = (int32_t)((uint32_t)s.n / (uint32_t)s.k);
  s.cA = s.n - s.k * s.a;
  s.cB = s.k - s.cA;
  return s;
}

// Block-wide exclusive scans of NV int64 values per thread in one pass (one
// set of barriers).  `scratch` holds 32 * (NV + 1) int64.  res[v] gets the
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

// Item fields (tile pairs U, live blocks n) of the first kPlanSmemItems items
// are staged in dynamic shared memory; later items are re-read from the item
// table.
constexpr int kPlanSmemItems = 24576;
constexpr int kKeyBits = 9;          // piece lengths 0..256 (and 257 as a query)
constexpr int32_t kNoKey = 511;      // lanes past the warp's items

size_t plan_smem_bytes(int64_t n_items) {
  const int64_t c = n_items < kPlanSmemItems ? n_items : kPlanSmemItems;
  return (size_t)(c * 6 + 16);
}

// The piece order is a stable counting sort of all pieces by length, longest
// first; inside a length, pieces follow their item, then tile pair, then
// their place in the item's split.  Warp w owns the contiguous item range
// [w R, (w + 1) R) (R = ceil(items / 32)) and walks it 32 items at a time, so
// item order is (warp, step, lane) order:
//   pass 2  per (warp, length) piece counts, per-warp unit / slot / combine
//           totals;
//   scan    bucket starts (lengths descending), per-(warp, length) offsets
//           (warps ascending), per-warp slot and combine bases;
//   pass 3  each warp places its pieces with no block barrier: a piece's
//           rank inside its length is the warp's running cursor for that
//           length plus the weights of earlier lanes of the same step with
//           that length, taken by pointer jumping over lanes of equal keys.
__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const MetaParams p, int32_t cached) {
  extern __shared__ __align__(16) unsigned char plan_dyn[];
  __shared__ int64_t scratch[32 * 5];
  __shared__ int64_t part[kPlanWarps][3];          // per warp: units, slots, combine records
  __shared__ int32_t bucket_start[kNumKeys];
  __shared__ int32_t warp_key[kPlanWarps][kNumKeys];  // counts, then running cursors
  __shared__ int64_t cost_sh[kPlanWarps];
  __shared__ int32_t abort_sh;
  int32_t* sU = reinterpret_cast<int32_t*>(plan_dyn);
  uint16_t* sN = reinterpret_cast<uint16_t*>(sU + cached);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < kPlanWarps * kNumKeys; i += blockDim.x) (&warp_key[0][0])[i] = 0;
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

  // stage the fields, total cost
  if (tid == 0) abort_sh = (meta[H_STATUS] & kDevBadSeqlen) ? 1 : 0;
  int64_t cost = 0;
#pragma unroll 4
  for (int32_t i = tid; i < n_items; i += kPlanThreads) {
    // item rows are 8 words on a 16-byte boundary: (.., n, n_tiles, ..)
    const int4 r = *reinterpret_cast<const int4*>(items + 8 * (int64_t)i);
    const int32_t U = (r.z + 1) / 2;
    if (i < cached) {
      sU[i] = U;
      sN[i] = (uint16_t)r.y;
    }
    cost += (int64_t)U * r.y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cost += __shfl_xor_sync(0xffffffffu, cost, o);
  if (lane == 0) cost_sh[warp] = cost;
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
  cost = 0;
  for (int w = 0; w < kPlanWarps; w++) cost += cost_sh[w];
  int64_t L64;
  if (p.forced_split > 0) {
    L64 = p.forced_split;
  } else {
    L64 = cdiv64(cost, 4LL * p.num_ctas);
    if (L64 < kMinSplitLen) L64 = kMinSplitLen;
  }
  if (L64 > 0x7fffffffLL) L64 = 0x7fffffffLL;
  const int32_t L = (int32_t)L64;
  if (tid == 0) {
    meta[H_SPLIT_LEN] = L;
    meta[H_COST_LO] = (int32_t)(uint32_t)(cost & 0xffffffffLL);
    meta[H_COST_HI] = (int32_t)(uint32_t)((uint64_t)cost >> 32);
  }

  const int32_t R = (n_items + kPlanWarps - 1) / kPlanWarps;
  const int32_t lo = warp * R < n_items ? warp * R : n_items;
  const int32_t hi = lo + R < n_items ? lo + R : n_items;

  // pass 2: per (warp, length) counts and per-warp totals
  {
    int64_t units = 0, slots = 0, combs = 0;
    for (int32_t i = lo + lane; i < hi; i += 32) {
      int32_t U, n;
      fields(i, U, n);
      const PieceShape s = piece_shape(U, n, L);
      atomicAdd(&warp_key[warp][s.a], s.U * s.cB);  // cB >= 1
      if (s.cA) atomicAdd(&warp_key[warp][s.a + 1], s.U * s.cA);
      units += (int64_t)s.U * s.k;
      if (s.k > 1) {
        slots += (int64_t)s.U * s.k;
        combs += s.U;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      units += __shfl_xor_sync(0xffffffffu, units, o);
      slots += __shfl_xor_sync(0xffffffffu, slots, o);
      combs += __shfl_xor_sync(0xffffffffu, combs, o);
    }
    if (lane == 0) {
      part[warp][0] = units;
      part[warp][1] = slots;
      part[warp][2] = combs;
    }
  }
  __syncthreads();

  // per length: offsets over warps (in place) and the length's total;
  // thread j holds length kNumKeys - 1 - j so that one scan over threads
  // gives the bucket starts longest first.  Threads 0..31 also carry warp
  // j's unit / slot / combine totals.
  int64_t n_units, n_slots, n_comb;
  {
    const int key = kNumKeys - 1 - tid;
    int64_t v[4] = {0, 0, 0, 0};
    if (tid < kNumKeys) {
      int32_t acc = 0;
      for (int w = 0; w < kPlanWarps; w++) {
        const int32_t c = warp_key[w][key];
        warp_key[w][key] = acc;
        acc += c;
      }
      v[0] = acc;
    }
    if (tid < kPlanWarps) {
      v[1] = part[tid][0];
      v[2] = part[tid][1];
      v[3] = part[tid][2];
    }
    int64_t r[4], t[4];
    block_exclusive_scan_n<4>(v, scratch, r, t);
    if (tid < kNumKeys) bucket_start[key] = (int32_t)r[0];
    if (tid < kPlanWarps) {
      part[tid][1] = r[2];
      part[tid][2] = r[3];
    }
    n_units = t[1];
    n_slots = t[2];
    n_comb = t[3];
  }
  if (tid == 0) {
    const bool over = n_units > g.unit_cap || n_slots > g.slot_cap || n_comb > g.comb_cap;
    meta[H_NUNITS] = over ? 0 : (int32_t)n_units;
    meta[H_NSLOTS] = over ? 0 : (int32_t)n_slots;
    meta[H_NCOMB] = over ? 0 : (int32_t)n_comb;
    if (over) raise_status(p, kDevCapacity);
  }
  __syncthreads();
  if (n_units > g.unit_cap || n_slots > g.slot_cap || n_comb > g.comb_cap) return;

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
    // slots and combine records in item order
    int32_t my_slots = s.k > 1 ? s.U * s.k : 0, my_combs = s.k > 1 ? s.U : 0;
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
    const int32_t slot_base = slot_cur + iS - my_slots;
    const int32_t comb_base = comb_cur + iC - my_combs;
    slot_cur += __shfl_sync(0xffffffffu, iS, 31);
    comb_cur += __shfl_sync(0xffffffffu, iC, 31);
    int32_t startA = 0, startB = 0;
    if (valid) {
      startB = bucket_start[a] + warp_key[warp][a] + preB;
      if (s.cA) startA = bucket_start[a + 1] + warp_key[warp][a + 1] + preA;
    }
    __syncwarp();
    // the last lane of each key group advances the warp's cursors
    if (valid && !(same & gt)) {
      atomicAdd(&warp_key[warp][a], sB);
      if (sA) atomicAdd(&warp_key[warp][a + 1], sA);
    }
    __syncwarp();
    if (valid) {
      if (s.k > 1)
        for (int32_t tp = 0; tp < s.U; tp++)
          comb[comb_base + tp] = make_int4(i, tp, slot_base + tp * s.k, s.k);
      int32_t j0 = 0, longs = 0;
      for (int32_t q = 0; q < s.k; q++) {
        const int32_t j1 = (int32_t)((uint32_t)((q + 1) * s.n) / (uint32_t)s.k);
        const bool is_long = j1 - j0 == s.a + 1 && s.cA;
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

cudaError_t launch_metadata(const MetaParams& p, cudaStream_t stream) {
  seq_kernel<<<1, kSeqThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t blocks = (p.geo.n_items + kItemWarps - 1) / kItemWarps;
  e = launch_dependent(item_kernel, dim3((unsigned)blocks), dim3(kItemWarps * 32), 0, stream, p);
  if (e != cudaSuccess) return e;
  const int32_t cached = p.geo.n_items < kPlanSmemItems ? p.geo.n_items : kPlanSmemItems;
  const size_t smem = plan_smem_bytes(p.geo.n_items);
  static int configured_device = -1;
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)plan_smem_bytes(kPlanSmemItems));
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  return launch_dependent(plan_kernel, dim3(1), dim3(kPlanThreads), smem, stream, p, cached);
}

}  // namespace gbsa
