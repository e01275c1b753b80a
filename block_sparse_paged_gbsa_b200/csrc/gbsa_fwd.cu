// gbsa_fwd.cu -- forward kernel of block-sparse paged GQA attention for
// sm_100a, and the split-KV combine kernel.
//
// Operation (GBSA article, cf-1.com/news/4865651, "Function / sparse
// attention mechanism"): out = Softmax(scale * Q * K_sparse^T + mask) *
// V_sparse, where each Q block of each KV head attends only to the KV blocks
// of its list, gathered from the paged cache (PA_BBND) through the block
// table.  Scores are produced tile by tile with the online softmax of the FA
// blog (ai6s.net), "three steps": running max, running sum and a rescale of
// the partial output, so the score matrix never exists.
//
// Design (one persistent CTA per SM, 512 threads, four warpgroups):
//   warps 0..3    softmax of tile 0 (TMEM lanes = tile rows)
//   warps 4..7    softmax of tile 1
//   warps 8..11   epilogue: O / l -> out (bf16, or fp16 for fp16 inputs)
//                 and lse, or split partials
//   warp 12       MMA issuer: S = Q K^T (SS MMA), O += P V (TS MMA, P read
//                 from TMEM); zeroes V rows of a last page past seqused_kv
//   warp 13       TMA producer: Q tiles and, per live block, the K and V
//                 pages into a ring of 5 x 32 KiB (10 x 16 KiB for E4M3)
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each; P overwrites
// the first columns of its S (two 16-bit or four E4M3 weights per column).
// Element types (kDt): bf16, fp16 (kind::f16 MMAs) and E4M3 (kind::f8f6f4,
// per-tensor dequantization scales folded into the score scale and 1 / l).
// Units come from the metadata work list, longest first: CTA c starts with
// unit c and then takes the next untaken unit from a counter in the work
// list's header, so SMs that run faster take more units.  Every wait is
// bounded (by FwdParams::wait_limit_ns, 1 s unless the caller sets another):
// after it the kernel sets GBSA_DEV_TIMEOUT, drains its own copies and MMAs
// (each drain bounded by 1 s), frees TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "gbsa_internal.cuh"
#include "sm100.cuh"

namespace gbsa {

using namespace sm100;

namespace {

constexpr int kThreads = 512;
// Register split: launched with kLaunchRegs per thread; the epilogue and
// control warpgroups give registers to the two softmax warpgroups.
constexpr int kLaunchRegs = 128;
// The instantiation with units in halves (below) moves 8 registers from each
// softmax thread to the MMA and producer warps, whose loop then carries both
// unit layouts.
template <bool kHalves>
constexpr int regs_softmax() { return kHalves ? 168 : 176; }  // warpgroups 0, 1
constexpr int kRegsEpilogue = 80;                              // warpgroup 2
template <bool kHalves>
constexpr int regs_control() { return kHalves ? 96 : 80; }    // warpgroup 3 (MMA, producer)
static_assert(256 * regs_softmax<false>() + 128 * kRegsEpilogue + 128 * regs_control<false>() <=
                  kLaunchRegs * kThreads,
              "register split exceeds the launch allocation");
static_assert(256 * regs_softmax<true>() + 128 * kRegsEpilogue + 128 * regs_control<true>() <=
                  kLaunchRegs * kThreads,
              "register split exceeds the launch allocation");
constexpr int kWarpMma = 12;
constexpr int kWarpProducer = 13;
constexpr int kStages = 5;
constexpr int kTileBytes = 32768;  // 128 rows x 128 16-bit elements (two SW128 boxes)
constexpr int kHalfBytes = 16384;
constexpr int kSmemQ = 0;
constexpr int kSmemRing = 2 * kTileBytes;
constexpr int kSmemBars = kSmemRing + kStages * kTileBytes;
// Bound of the final drains (the copies and MMAs a CTA issued must land
// before it exits); the pipeline waits use FwdParams::wait_limit_ns.
constexpr uint64_t kWaitLimitNs = 1000000000ull;
// A unit whose item has a single tile (decode: one token x G heads) and at
// least this many blocks runs in halves: both tile slots work on its even /
// odd blocks, so the S -> softmax -> PV chain of one slot overlaps the other.
// Only the kernel instantiated with kHalves (chosen by the host when every Q
// block fits one tile) carries this code: in the other one its extra branch
// on the MMA warp costs the two-tile units a few percent.
// Items with more tiles keep their last odd tile on one slot: that unit reads
// the same K/V as the item's two-tile unit on another SM, and in step with it
// one of the two finds the pages in L2 (in halves it runs ahead and both miss).
#ifndef GBSA_HALVES_MIN_BLOCKS
#define GBSA_HALVES_MIN_BLOCKS 4
#endif
constexpr int32_t kHalvesMinBlocks = GBSA_HALVES_MIN_BLOCKS;
static_assert(kHalvesMinBlocks >= 2, "a unit in halves needs a block per slot");
// Element types of Q, K, V (and P): 0 = bf16, 1 = fp16, 2 = E4M3.  A D = 128
// row is two 64-element halves of 128 B for the 16-bit types and one 128 B
// half for E4M3; E4M3 MMAs (kind::f8f6f4) take K = 32 per instruction, so a
// block needs 4 instead of 8 per product.  The output is fp16 for fp16
// inputs and bf16 otherwise.
constexpr int kDtBf16 = 0, kDtFp16 = 1, kDtE4m3 = 2;
template <int kDt>
constexpr int d_halves() { return kDt == kDtE4m3 ? 1 : 2; }
// The K/V ring: kStages stages of a 16-bit block (32 KiB), or twice as many
// E4M3 blocks (16 KiB) in the same bytes, so that as many bytes stay in
// flight per SM (decode is bound by that, not by the arithmetic).
constexpr int kMaxStages = 2 * kStages;
template <int kDt>
constexpr int ring_stages() { return kStages * 2 / d_halves<kDt>(); }
template <int kDt>
constexpr int stage_bytes() { return kHalfBytes * d_halves<kDt>(); }
// Instruction descriptors: S = Q K^T (K-major A and B), O += P V (V MN-major),
// fp32 accumulator.  E4M3 and fp16 share the format code 0.
template <int kDt>
constexpr uint32_t idesc_qk() {
  return kDt == kDtBf16 ? idesc_bf16_f32(128, 128, false, false)
                        : idesc_f16_f32(128, 128, false, false);
}
template <int kDt>
constexpr uint32_t idesc_pv() {
  return kDt == kDtBf16 ? idesc_bf16_f32(128, 128, false, true)
                        : idesc_f16_f32(128, 128, false, true);
}
// Lazy-rescale threshold (log2 units).  16-bit P: the reference max may lag
// the row max by up to 8 (P <= 256).  E4M3 P is formed as 2^8 * p so that the
// small weights stay above its 2^-9 floor; the reference may then lag by 0.5
// at most (P <= 362 < 448, the largest E4M3 value).
template <int kDt>
constexpr float rescale_threshold() { return kDt == kDtE4m3 ? 0.5f : 8.0f; }

// A score held as a float, or as the raw 32-bit word a TMEM load gives.
__device__ __forceinline__ float as_float(float x) { return x; }
__device__ __forceinline__ float as_float(uint32_t x) { return __uint_as_float(x); }

struct FwdParams {
  const int32_t* meta;
  int32_t* work;  // meta + H_UNIT_NEXT: the unit counter, then the finished-CTA count
  const int32_t* block_table;  // paged K/V
  const int64_t* cu_kv;        // TND K/V: first row of each sequence (block_table unused)
  uint16_t* out;  // fp16 for fp16 inputs, else bf16
  float* lse;
  float* ws_o;    // [slot_cap][rows_per_unit][128] fp32 partial outputs
  float* ws_lse;  // [slot_cap][rows_per_unit] fp32 partial lse
  int32_t* dev_status;
  uint32_t signature;
  int32_t N1, N2, G, T, top_k, max_pages, num_pages, tile_tokens, rows_per_unit;
  int32_t win_left, return_lse;
  float scale_log2;  // softmax scale (E4M3: times q_scale * k_scale) x log2(e)
  float out_scale;   // E4M3: v_scale
  uint64_t wait_limit_ns;  // bound of every pipeline wait
};

// The units a CTA takes after its first come from a counter shared by the
// grid (in list order, so a fast SM takes more units than a slow one).  Its
// producer warp fetches each one and hands the unit's record (its unit-table
// row and its item's row) to the other roles through a ring of kUnitQ entries.
constexpr uint32_t kUnitQ = 4;
constexpr uint32_t kUnitReaders = 13;  // warps 0..12: softmax 8, epilogue 4, MMA 1
struct UnitRec {
  int4 rec;   // unit row: item, tile pair, blocks [j0, j1), split slot
  int4 a, c;  // item row, words 0..3 and 4..7
};

struct Bars {
  UnitRec uq[kUnitQ];
  int32_t uq_id[kUnitQ];      // unit index, or -1: no more units
  uint64_t uq_full[kUnitQ];   // entry written (producer)
  uint64_t uq_empty[kUnitQ];  // entry read (one arrival per reading warp)
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[kMaxStages], kv_empty[kMaxStages];
  uint64_t s_full[2];      // S of a block ready (MMA commit)
  uint64_t p_full[2];      // P of a block in TMEM, O rescaled (128 softmax threads)
  uint64_t o_final[2];     // last PV of a unit complete (MMA commit)
  uint64_t o_free[2];      // epilogue has read O (128 epilogue threads)
  uint64_t stats_full[2];  // row max / sum of a unit in `stats` (128 softmax threads)
  uint64_t stats_free[2];  // epilogue has read them (128 epilogue threads)
  uint64_t drain;
  uint64_t wait_limit_ns;  // FwdParams::wait_limit_ns, read on the slow path of a wait
  uint32_t tmem_base;
  int32_t abort;
  float2 stats[2][128];    // (reference max in log2 units, row sum) per tile row
};
constexpr int kSmemBytes = kSmemBars + (int)sizeof(Bars);
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Unit {
  int32_t item, tp, j0, j1, slot;
  int32_t b, n_tiles, tok_begin, n_store, n_used, pos0, ku;
  int32_t kvh, nt;  // KV head, tiles in this unit (1 or 2)
  bool halves;      // one tile, >= 2 blocks: the two tile slots take its even
                    // and odd blocks (two partial softmaxes, merged at the end)
};

// The record of unit u, read from the work list in global memory.
__device__ __forceinline__ UnitRec fetch_unit(const int32_t* meta, int64_t off_unit,
                                              int64_t off_item, int32_t u) {
  UnitRec r;
  r.rec = *reinterpret_cast<const int4*>(meta + off_unit + 4 * (int64_t)u);
  r.a = *reinterpret_cast<const int4*>(meta + off_item + 8 * (int64_t)r.rec.x);
  r.c = *reinterpret_cast<const int4*>(meta + off_item + 8 * (int64_t)r.rec.x + 4);
  return r;
}

template <bool kHalves>
__device__ __forceinline__ Unit decode_unit(const UnitRec& r, int32_t N2) {
  Unit x;
  const int4 rec = r.rec, a = r.a, c = r.c;
  x.item = rec.x;
  x.tp = rec.y;
  x.j0 = rec.z & 0xffff;
  x.j1 = (int32_t)((uint32_t)rec.z >> 16);
  x.slot = rec.w;
  x.b = a.x;
  x.n_tiles = a.z;
  x.tok_begin = a.w;
  x.n_store = c.x;
  x.n_used = c.y;
  x.pos0 = c.z;
  x.ku = c.w;
  x.kvh = x.item % N2;
  x.nt = min(2, x.n_tiles - 2 * x.tp);
  x.halves = kHalves && x.n_tiles == 1 && x.j1 - x.j0 >= kHalvesMinBlocks;
  return x;
}

// Bounded wait on an mbarrier phase.  Returns false (and raises the CTA's
// abort flag) after the pipeline wait limit, or at once if another role
// aborted.  The clock starts after the first probe, which the hardware may
// hold for a while on its own: a wait gives up no earlier than the limit.
// (A 1 us suspend hint on every probe made the limit tight but cost decode
// 4.5 %: the waiting warps woke and polled far more often.)
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Bars* bars) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; i++)
      if (mbar_try_wait(bar, parity)) return true;
    if (*reinterpret_cast<volatile int32_t*>(&bars->abort)) return false;
    if (global_timer_ns() - t0 > bars->wait_limit_ns) {
      atomicExch(&bars->abort, 1);
      return false;
    }
  }
}

// The k-th entry of the unit queue, read by a whole warp: waits until the
// producer wrote it, copies it, and (lane 0, once every lane has read it)
// releases it.  False when the queue has ended (unit < 0) or a wait gave up.
struct UnitCursor {
  uint32_t k = 0;
  __device__ __forceinline__ bool next(Bars* bars, UnitRec& r) {
    const uint32_t s = k % kUnitQ;
    if (!wait_bar(&bars->uq_full[s], (k / kUnitQ) & 1, bars)) return false;
    const int32_t u = bars->uq_id[s];
    r = bars->uq[s];
    __syncwarp();
    if (lane_id() == 0) mbar_arrive(&bars->uq_empty[s]);
    k++;
    return u >= 0;
  }
};

// Producer side: writes unit u (u < 0: the end) as the k-th entry once every
// reader has released the entry's previous use.  Whole warp; lane 0 writes.
__device__ __forceinline__ bool push_unit(Bars* bars, uint32_t k, int32_t u, const UnitRec& r,
                                          uint32_t lane) {
  const uint32_t s = k % kUnitQ;
  if (k >= kUnitQ && !wait_bar(&bars->uq_empty[s], ((k / kUnitQ) & 1) ^ 1, bars)) return false;
  if (lane == 0) {
    bars->uq[s] = r;
    bars->uq_id[s] = u;
    mbar_arrive(&bars->uq_full[s]);
  }
  return true;
}

// Operand layouts in shared memory (128-byte swizzle, tiles 1 KiB aligned):
//   Q and K tiles, K-major: 128 rows x 128 B per 64-column half, halves
//   16 KiB apart; a K step of 16 16-bit elements advances 32 B inside the
//   row.  E4M3: one half of 128 columns, a K step of 32 elements (32 B).
//   V tile, MN-major (N = D): the two 64-column halves of D 16 KiB apart
//   (leading byte offset), 8-key groups 1 KiB apart; a K step of 16 keys
//   advances 2 KiB (E4M3: D in one 128 B row, a K step of 32 keys 4 KiB).

// Row identity of TMEM lane `row` in tile `slot` of unit x.
struct RowInfo {
  bool store;   // row holds a stored query token of this unit (out is written)
  bool used;    // ... and the token is used (t < seqused_q)
  int32_t tok;  // global token index
  int32_t h;    // query head
  int32_t pos;  // query position (bottom-right aligned causal)
};

__device__ __forceinline__ RowInfo row_info(const FwdParams& p, const Unit& x, int slot, int row) {
  RowInfo r;
  const int rows_in_tile = p.tile_tokens * p.G;
  const int tok_in_tile = row / p.G;
  const int32_t tok_off = (2 * x.tp + slot) * p.tile_tokens + tok_in_tile;
  r.store = row < rows_in_tile && tok_off < x.n_store;
  r.used = r.store && tok_off < x.n_used;
  r.tok = x.tok_begin + tok_off;
  r.h = x.kvh * p.G + (row - tok_in_tile * p.G);
  r.pos = x.pos0 + tok_off;
  return r;
}

// ---------------------------------------------------------------------------
// producer (one thread)
// ---------------------------------------------------------------------------
// Called by the whole producer warp: every lane waits and counts, lane 0
// issues the copies.  `where` is the physical page (paged pool: 4-D map) or,
// with `tnd`, the first row of the block in k / v [T_kv, N2, D] (3-D map).
// A block is d_halves<kDt>() boxes of 128 rows x 128 B (64 elements of a
// 16-bit type, or 128 E4M3 elements).
template <int kDt>
__device__ __forceinline__ bool produce_kv(const CUtensorMap* map, uint8_t* smem, Bars* bars,
                                           uint32_t& kv_iter, int32_t kvh, int32_t where,
                                           bool tnd, uint32_t lane) {
  constexpr uint32_t kN = ring_stages<kDt>();
  const uint32_t stage = kv_iter % kN;
  if (kv_iter >= kN && !wait_bar(&bars->kv_empty[stage], ((kv_iter / kN) & 1) ^ 1, bars))
    return false;
  if (lane == 0) {
    uint8_t* dst = smem + kSmemRing + stage * stage_bytes<kDt>();
    mbar_arrive_expect_tx(&bars->kv_full[stage], d_halves<kDt>() * kHalfBytes);
#pragma unroll
    for (int h = 0; h < d_halves<kDt>(); h++) {
      if (tnd)
        tma_load_3d(dst + h * kHalfBytes, map, &bars->kv_full[stage], 64 * h, kvh, where);
      else
        tma_load_4d(dst + h * kHalfBytes, map, &bars->kv_full[stage], 64 * h, kvh, 0, where);
    }
  }
  kv_iter++;
  return true;
}

template <int kDt>
__device__ __forceinline__ bool produce_q(const FwdParams& p, const CUtensorMap* map_q,
                                          uint8_t* smem, Bars* bars, uint32_t& q_iter,
                                          const Unit& x, int s, uint32_t lane) {
  if (q_iter > 0 && !wait_bar(&bars->q_empty[s], (q_iter - 1) & 1, bars)) return false;
  if (lane == 0) {
    const uint32_t box_bytes = 128u * (uint32_t)p.G * (uint32_t)p.tile_tokens;
    const int32_t tok = x.tok_begin + (2 * x.tp + s) * p.tile_tokens;
    uint8_t* dst = smem + kSmemQ + s * kTileBytes;
    mbar_arrive_expect_tx(&bars->q_full[s], (uint32_t)d_halves<kDt>() * box_bytes);
#pragma unroll
    for (int h = 0; h < d_halves<kDt>(); h++)
      tma_load_3d(dst + h * kHalfBytes, map_q, &bars->q_full[s], 64 * h, x.kvh * p.G, tok);
  }
  q_iter++;
  return true;
}

// The copies of one unit with n > 0 blocks (whole warp; lane 0 issues).
template <bool kHalves, int kDt>
__device__ __forceinline__ void produce_unit(const FwdParams& p, const CUtensorMap* map_q,
                                             const CUtensorMap* map_k, const CUtensorMap* map_v,
                                             uint8_t* smem, Bars* bars, const Unit& x,
                                             int64_t off_list, uint32_t& kv_iter,
                                             uint32_t& q_iter0, uint32_t& q_iter1, int32_t& bad,
                                             bool& ok, uint32_t lane) {
  const int32_t n = x.j1 - x.j0;
  const int32_t* list = p.meta + off_list + (int64_t)x.item * p.top_k + x.j0;
  const bool tnd = p.cu_kv != nullptr;
  const int32_t* bt = tnd ? nullptr : p.block_table + (int64_t)x.b * p.max_pages;
  const int64_t row0 = tnd ? p.cu_kv[x.b] : 0;  // TND: first row of the sequence
  // order: Q0, K_0, Q1, V_0, K_1, V_1, ... (Q1 of a unit waits for the
  // previous unit's last S1, which comes later than its last S0); a unit
  // in halves: Q0, then per block pair K_j, K_j+1, V_j, V_j+1
  // pages of the first 32 entries: the loads overlap the wait for the Q slot
  // per lane: the page of an entry (paged), or its first row (TND); live
  // entries lie inside the sequence, so a TND row stays inside k / v
  int32_t page = 0;
  if ((int32_t)lane < n) {
    const int32_t lb = list[lane] & kEntryLbMask;
    page = tnd ? (int32_t)(row0 + (int64_t)lb * kPage) : (lb < p.max_pages ? bt[lb] : -1);
  }
  ok = produce_q<kDt>(p, map_q, smem, bars, q_iter0, x, 0, lane);
  for (int32_t c0 = 0; c0 < n && ok; c0 += 32) {
    if (c0 > 0 && c0 + (int32_t)lane < n) {
      const int32_t lb = list[c0 + lane] & kEntryLbMask;
      page = tnd ? (int32_t)(row0 + (int64_t)lb * kPage) : (lb < p.max_pages ? bt[lb] : -1);
    }
    if (!tnd && c0 + (int32_t)lane < n && (page < 0 || page >= p.num_pages)) {
      bad |= kDevBadPage;
      page = 0;
    }
    const int32_t cn = min(32, n - c0);
    if (x.halves) {
      // blocks c0 + jj (even) and c0 + jj + 1 share a 32-entry chunk
      for (int32_t jj = 0; jj < cn && ok; jj += 2) {
        const bool has1 = jj + 1 < cn;
        const int32_t pg0 = __shfl_sync(0xffffffffu, page, jj);
        const int32_t pg1 = __shfl_sync(0xffffffffu, page, (jj + 1) & 31);
        ok = produce_kv<kDt>(map_k, smem, bars, kv_iter, x.kvh, pg0, tnd, lane);
        if (ok && has1) ok = produce_kv<kDt>(map_k, smem, bars, kv_iter, x.kvh, pg1, tnd, lane);
        if (ok) ok = produce_kv<kDt>(map_v, smem, bars, kv_iter, x.kvh, pg0, tnd, lane);
        if (ok && has1) ok = produce_kv<kDt>(map_v, smem, bars, kv_iter, x.kvh, pg1, tnd, lane);
      }
      continue;
    }
    for (int32_t jj = 0; jj < cn && ok; jj++) {
      const int32_t pg = __shfl_sync(0xffffffffu, page, jj);
      ok = produce_kv<kDt>(map_k, smem, bars, kv_iter, x.kvh, pg, tnd, lane);
      if (ok && c0 + jj == 0 && x.nt == 2) ok = produce_q<kDt>(p, map_q, smem, bars, q_iter1, x, 1, lane);
      if (ok) ok = produce_kv<kDt>(map_v, smem, bars, kv_iter, x.kvh, pg, tnd, lane);
    }
  }
}

template <bool kHalves, int kDt>
__device__ void run_producer(const FwdParams& p, const CUtensorMap* map_q, const CUtensorMap* map_k,
                             const CUtensorMap* map_v, uint8_t* smem, Bars* bars, int32_t n_units,
                             int64_t off_unit, int64_t off_item, int64_t off_list) {
  // The whole warp runs the loop: lanes resolve 32 list entries and their
  // physical pages in parallel (two dependent loads per 32 blocks instead of
  // per block); lane 0 issues the copies.
  const uint32_t lane = lane_id();
  uint32_t kv_iter = 0, q_iter0 = 0, q_iter1 = 0;
  int32_t bad = 0;
  bool ok = true;
  // the first unit of CTA c is unit c; the next ones come from the counter
  int32_t u = (int32_t)blockIdx.x;
  for (uint32_t kq = 0; ok; kq++) {
    const bool live = u < n_units;
    UnitRec r{};
    if (live) r = fetch_unit(p.meta, off_unit, off_item, u);
    const Unit x = decode_unit<kHalves>(r, p.N2);
    const int32_t n = x.j1 - x.j0;
    if (!(ok = push_unit(bars, kq, live ? u : -1, r, lane))) break;
    if (!live) break;
    // the unit after this one; the atomic's latency overlaps this unit's
    // copies, and its value is always read (below) so that it has completed
    // before the CTA counts itself finished
    int32_t nxt = 0;
    if (lane == 0) nxt = (int32_t)gridDim.x + atomicAdd(p.work, 1);
    if (n > 0) produce_unit<kHalves, kDt>(p, map_q, map_k, map_v, smem, bars, x, off_list, kv_iter,
                                          q_iter0, q_iter1, bad, ok, lane);
    u = __shfl_sync(0xffffffffu, nxt, 0);
  }
  if (lane == 0) {
    // This CTA fetches no more units (after an abort too): it counts itself,
    // and the last CTA to do so puts both counters back to zero for the next
    // launch on this work list.  Every CTA counts itself only after the value
    // of its last fetch came back, so no fetch follows the reset.  (Counting
    // here, not at the CTA's exit, keeps the atomics off the exit path.)
    __threadfence();
    if (atomicAdd(p.work + 1, 1) == min((int32_t)gridDim.x, n_units) - 1) {
      atomicExch(p.work, 0);
      atomicExch(p.work + 1, 0);
    }
  }
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (lane == 0 && bad && p.dev_status) atomicOr(p.dev_status, bad);
  if (!ok && lane == 0) {
    // drain: wait (bounded) for the copies this thread issued last
    const uint64_t t0 = global_timer_ns();
    constexpr uint32_t kN = ring_stages<kDt>();
    for (uint32_t i = (kv_iter > kN ? kv_iter - kN : 0); i < kv_iter; i++) {
      while (!mbar_try_wait(&bars->kv_full[i % kN], (i / kN) & 1) &&
             global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
    if (q_iter0 > 0)
      while (!mbar_try_wait(&bars->q_full[0], (q_iter0 - 1) & 1) &&
             global_timer_ns() - t0 < kWaitLimitNs) {
      }
    if (q_iter1 > 0)
      while (!mbar_try_wait(&bars->q_full[1], (q_iter1 - 1) & 1) &&
             global_timer_ns() - t0 < kWaitLimitNs) {
      }
  }
}

// ---------------------------------------------------------------------------
// MMA issuer (one warp; lane 0 waits and issues, the warp zeroes stale V rows)
//
// Issue order for a two-tile unit with blocks 0..n-1 (tcgen05 MMAs of a CTA
// execute in issue order, so an S written after the PV that reads the P
// aliased on it needs no wait):
//     S0_0, S1_0, PV0_0,
//     for i >= 1:  S0_i, PV1_{i-1}, S1_i, PV0_i,
//     PV1_{n-1}.
// While softmax 0 works on S0_i the tensor pipe runs PV1_{i-1} and S1_i, and
// while softmax 1 works on S1_i it runs PV0_i and S0_{i+1}.  K_i is released
// after S1_i, V_i after PV1_i, which keeps the ring in fill order.
// ---------------------------------------------------------------------------
// Warp-wide wait: every lane polls the barrier.  One lane polling while the
// rest wait at a shuffle costs ~300 cycles per wait in a warp that issues
// tcgen05 MMAs (the pipe drains meanwhile); all lanes polling costs ~20.  The
// lanes execute each try_wait, abort read and timer read together, so they
// agree on the result.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Bars* bars) {
  return wait_bar(bar, parity, bars);
}

// Descriptors are handled as 32-bit low words (start address >> 4 in bits
// [0,14), leading byte offset >> 4 in [16,30)) plus the shared high word;
// offsets are added to the low word (addresses stay below 256 KiB: no carry).
template <int kDt>
__device__ __forceinline__ void issue_qk(uint32_t d_tmem, uint32_t q_lo, uint32_t k_lo,
                                         uint32_t hi) {
  if constexpr (kDt == kDtE4m3) {
#pragma unroll
    for (int kk = 0; kk < 4; kk++) {  // 32 E4M3 elements (32 B) per step, one 128 B half
      const uint32_t off = (kk * 32) >> 4;
      mma_ss_lo_f8(d_tmem, q_lo + off, k_lo + off, hi, idesc_qk<kDt>(), kk > 0 ? 1u : 0u);
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < 8; kk++) {
      const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
      mma_ss_lo(d_tmem, q_lo + off, k_lo + off, hi, idesc_qk<kDt>(), kk > 0 ? 1u : 0u);
    }
  }
}

template <int kDt>
__device__ __forceinline__ void issue_pv(uint32_t d_tmem, uint32_t p_tmem, uint32_t v_lo,
                                         uint32_t hi, bool accumulate) {
  if constexpr (kDt == kDtE4m3) {
    // P: 4 E4M3 per TMEM column, 32 keys (8 columns) per step; V: 32 keys of
    // 128 B per step
#pragma unroll
    for (int kk = 0; kk < 4; kk++)
      mma_ts_lo_f8(d_tmem, p_tmem + kk * 8, v_lo + ((kk * 4096) >> 4), hi, idesc_pv<kDt>(),
                   (accumulate || kk > 0) ? 1u : 0u);
  } else {
    // P: 2 elements per column, 16 keys (8 columns) per step; V: 16 keys of
    // two 128 B halves per step
#pragma unroll
    for (int kk = 0; kk < 8; kk++)
      mma_ts_lo(d_tmem, p_tmem + kk * 8, v_lo + ((kk * 2048) >> 4), hi, idesc_pv<kDt>(),
                (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Position in a K/V ring of kN stages: stage index and the parity of its
// current fill.
template <uint32_t kN>
struct RingPos {
  uint32_t stage, phase;
  __device__ __forceinline__ void advance() {
    if (++stage == kN) {
      stage = 0;
      phase ^= 1u;
    }
  }
  // the position k fills later (k < kN)
  __device__ __forceinline__ RingPos ahead(uint32_t k) const {
    RingPos r{stage + k, phase};
    if (r.stage >= kN) {
      r.stage -= kN;
      r.phase ^= 1u;
    }
    return r;
  }
};

// Zero the rows of a V tile that lie past seqused_kv on a last page (their
// pool contents are arbitrary and P there is 0, but 0 * NaN is NaN).  Whole
// warp; `entry` is the block's list entry.
template <int kDt>
__device__ __forceinline__ void zero_v_tail(uint8_t* smem, uint32_t vs, int32_t entry, int32_t ku,
                                            uint32_t lane) {
  if (!(entry & kEntryPartial)) return;
  const int32_t r0 = min(max(ku - (entry & kEntryLbMask) * kPage, 0), kPage);
  uint8_t* vt = smem + kSmemRing + vs * stage_bytes<kDt>();
  constexpr int32_t kChunks = 8 * d_halves<kDt>();  // 16-byte chunks of a row
  const int32_t n16 = (kPage - r0) * kChunks;
  for (int32_t t = lane; t < n16; t += 32) {
    const int32_t row = r0 + t / kChunks, chunk = t % kChunks;
    *reinterpret_cast<uint4*>(vt + (chunk >> 3) * kHalfBytes + row * 128 + (chunk & 7) * 16) =
        make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  __syncwarp();
}

template <bool kHalves, int kDt>
__device__ void run_mma(const FwdParams& p, uint8_t* smem, Bars* bars, uint32_t tmem,
                        int64_t off_list) {
  const uint32_t lane = lane_id();
  uint32_t q_iter0 = 0, q_iter1 = 0;
  uint32_t blk0 = 0, blk1 = 0;      // blocks per tile slot (p_full phases)
  uint32_t units0 = 0, units1 = 0;  // units per tile slot (o_free phases)
  using Ring = RingPos<ring_stages<kDt>()>;
  Ring rp{0, 0};                    // next K/V tile to consume
  bool ok = true;
  const uint32_t q_addr = smem_u32(smem + kSmemQ);
  const uint32_t ring_addr = smem_u32(smem + kSmemRing);
  const uint64_t d0 = smem_desc_sw128(q_addr, 16, 1024);
  const uint32_t hi = (uint32_t)(d0 >> 32);
  const uint32_t q0_lo = (uint32_t)d0;
  const uint32_t q1_lo = q0_lo + (kTileBytes >> 4);
  const uint32_t k_lo0 = (uint32_t)smem_desc_sw128(ring_addr, 16, 1024);
  const uint32_t v_lo0 = (uint32_t)smem_desc_sw128(ring_addr, kHalfBytes, 1024);
  constexpr uint32_t kStageLo = stage_bytes<kDt>() >> 4;

  UnitRec ur;
  for (UnitCursor cur; ok && cur.next(bars, ur);) {
    const int4 rec = ur.rec, irow = ur.a;
    const int32_t item = rec.x, j0 = rec.z & 0xffff, n = (int32_t)((uint32_t)rec.z >> 16) - j0;
    const int32_t ku = ur.c.w;
    const bool two = irow.z - 2 * rec.y >= 2;
    const bool halves = kHalves && irow.z == 1 && n >= kHalvesMinBlocks;
    if (halves) {
      // One tile, its blocks split even (slot 0) / odd (slot 1); both S read
      // Q0.  Ring order per block pair j, j+1: K_j, K_j+1, V_j, V_j+1, each
      // released right after the MMA that reads it.
      //     S0_0, S1_0, PV0_0, then for i >= 1: S0_i, PV1_{i-1}, S1_i, PV0_i,
      //     and PV1 of the last odd block when n is even.
      const int32_t* list = p.meta + off_list + (int64_t)item * p.top_k + j0;
      int32_t entries = (int32_t)lane < n ? list[lane] : 0;
      if (!(ok = warp_wait(&bars->q_full[0], q_iter0 & 1, bars))) break;
      q_iter0++;
      const int32_t n0 = (n + 1) >> 1, n1 = n >> 1;
      // blocks of these 32 whose V tile has rows past seqused_kv (bit j & 31):
      // a register test per block instead of a shuffle of the entry
      uint32_t partial = __ballot_sync(0xffffffffu, entries & kEntryPartial);
      uint32_t pv1 = 0;  // ring stage of V of the pending odd block
      for (int32_t i = 0; i < n0 && ok; i++) {
        const int32_t j = 2 * i;
        const bool has1 = j + 1 < n;
        if (i > 0 && (j & 31) == 0) {
          entries = j + (int32_t)lane < n ? list[j + lane] : 0;
          partial = __ballot_sync(0xffffffffu, entries & kEntryPartial);
        }
        // ---- S0_i = Q K_j
        if (!(ok = warp_wait(&bars->kv_full[rp.stage], rp.phase, bars))) break;
        if (lane == 0) {
          tc_fence_after_sync();
          issue_qk<kDt>(tmem, q0_lo, k_lo0 + rp.stage * kStageLo, hi);
          tc_commit(&bars->s_full[0]);
          tc_commit(&bars->kv_empty[rp.stage]);
          if (j == n - 1) tc_commit(&bars->q_empty[0]);
        }
        // ---- PV1_{i-1} = P1 V_{j-1}
        if (i > 0) {
          if (i == 1 && units1 > 0)
            if (!(ok = warp_wait(&bars->o_free[1], (units1 - 1) & 1, bars))) break;
          if (!(ok = warp_wait(&bars->p_full[1], blk1 & 1, bars))) break;
          if (lane == 0) {
            tc_fence_after_sync();
            issue_pv<kDt>(tmem + 384, tmem + 128, v_lo0 + pv1 * kStageLo, hi, i - 1 > 0);
            if (i == n1) tc_commit(&bars->o_final[1]);
            tc_commit(&bars->kv_empty[pv1]);
          }
          blk1++;
        }
        // ---- S1_i = Q K_{j+1}
        if (has1) {
          const Ring rk1 = rp.ahead(1);
          if (!(ok = warp_wait(&bars->kv_full[rk1.stage], rk1.phase, bars))) break;
          if (lane == 0) {
            tc_fence_after_sync();
            issue_qk<kDt>(tmem + 128, q0_lo, k_lo0 + rk1.stage * kStageLo, hi);
            tc_commit(&bars->s_full[1]);
            tc_commit(&bars->kv_empty[rk1.stage]);
            if (j + 1 == n - 1) tc_commit(&bars->q_empty[0]);
          }
        }
        // ---- V_j, then PV0_i = P0 V_j
        const Ring rv0 = rp.ahead(has1 ? 2 : 1);
        if (!(ok = warp_wait(&bars->kv_full[rv0.stage], rv0.phase, bars))) break;
        if ((partial >> (j & 31)) & 1u)
          zero_v_tail<kDt>(smem, rv0.stage, __shfl_sync(0xffffffffu, entries, j & 31), ku, lane);
        if (i == 0 && units0 > 0)
          if (!(ok = warp_wait(&bars->o_free[0], (units0 - 1) & 1, bars))) break;
        if (!(ok = warp_wait(&bars->p_full[0], blk0 & 1, bars))) break;
        if (lane == 0) {
          tc_fence_after_sync();
          issue_pv<kDt>(tmem + 256, tmem, v_lo0 + rv0.stage * kStageLo, hi, i > 0);
          if (i == n0 - 1) tc_commit(&bars->o_final[0]);
          tc_commit(&bars->kv_empty[rv0.stage]);
        }
        blk0++;
        // ---- V_{j+1} (read by PV1_i)
        if (has1) {
          const Ring rv1 = rp.ahead(3);
          if (!(ok = warp_wait(&bars->kv_full[rv1.stage], rv1.phase, bars))) break;
          if ((partial >> ((j + 1) & 31)) & 1u)
            zero_v_tail<kDt>(smem, rv1.stage, __shfl_sync(0xffffffffu, entries, (j + 1) & 31), ku,
                             lane);
          pv1 = rv1.stage;
        }
        rp = rp.ahead(has1 ? 4 : 2);
      }
      // ---- PV1 of the last odd block when n is even
      if (ok && n1 == n0) {
        if (n1 == 1 && units1 > 0) ok = warp_wait(&bars->o_free[1], (units1 - 1) & 1, bars);
        if (ok) ok = warp_wait(&bars->p_full[1], blk1 & 1, bars);
        if (ok && lane == 0) {
          tc_fence_after_sync();
          issue_pv<kDt>(tmem + 384, tmem + 128, v_lo0 + pv1 * kStageLo, hi, n1 - 1 > 0);
          tc_commit(&bars->o_final[1]);
          tc_commit(&bars->kv_empty[pv1]);
        }
        blk1++;
      }
    } else if (n > 0) {
      // list entries of this unit, 32 at a time, one per lane (no global
      // load on the issue path); the load overlaps the wait for Q
      const int32_t* list = p.meta + off_list + (int64_t)item * p.top_k + j0;
      int32_t entries = (int32_t)lane < n ? list[lane] : 0;
      if (!(ok = warp_wait(&bars->q_full[0], q_iter0 & 1, bars))) break;
      q_iter0++;
      uint32_t prev_vs = 0;
      for (int32_t i = 0; i < n && ok; i++) {
        if (i > 0 && (i & 31) == 0) entries = i + (int32_t)lane < n ? list[i + lane] : 0;
        // ---- S0_i
        const uint32_t ks = rp.stage;
        if (!(ok = warp_wait(&bars->kv_full[ks], rp.phase, bars))) break;
        rp.advance();
        if (lane == 0) {
          tc_fence_after_sync();
          issue_qk<kDt>(tmem, q0_lo, k_lo0 + ks * kStageLo, hi);
          tc_commit(&bars->s_full[0]);
          if (i == n - 1) tc_commit(&bars->q_empty[0]);
        }
        if (two) {
          if (i == 0) {
            if (!(ok = warp_wait(&bars->q_full[1], q_iter1 & 1, bars))) break;
            q_iter1++;
          } else {
            // ---- PV1_{i-1}
            if (i == 1 && units1 > 0)
              if (!(ok = warp_wait(&bars->o_free[1], (units1 - 1) & 1, bars))) break;
            if (!(ok = warp_wait(&bars->p_full[1], blk1 & 1, bars))) break;
            if (lane == 0) {
              tc_fence_after_sync();
              issue_pv<kDt>(tmem + 384, tmem + 128, v_lo0 + prev_vs * kStageLo, hi, i - 1 > 0);
              tc_commit(&bars->kv_empty[prev_vs]);
            }
            blk1++;
          }
          // ---- S1_i
          if (lane == 0) {
            issue_qk<kDt>(tmem + 128, q1_lo, k_lo0 + ks * kStageLo, hi);
            tc_commit(&bars->s_full[1]);
            if (i == n - 1) tc_commit(&bars->q_empty[1]);
          }
        }
        if (lane == 0) tc_commit(&bars->kv_empty[ks]);
        // ---- V_i: zero the rows of a last page past seqused_kv
        const uint32_t vs = rp.stage;
        if (!(ok = warp_wait(&bars->kv_full[vs], rp.phase, bars))) break;
        rp.advance();
        zero_v_tail<kDt>(smem, vs, __shfl_sync(0xffffffffu, entries, i & 31), ku, lane);
        // ---- PV0_i
        if (i == 0 && units0 > 0)
          if (!(ok = warp_wait(&bars->o_free[0], (units0 - 1) & 1, bars))) break;
        if (!(ok = warp_wait(&bars->p_full[0], blk0 & 1, bars))) break;
        if (lane == 0) {
          tc_fence_after_sync();
          issue_pv<kDt>(tmem + 256, tmem, v_lo0 + vs * kStageLo, hi, i > 0);
          if (i == n - 1) tc_commit(&bars->o_final[0]);
          if (!two) tc_commit(&bars->kv_empty[vs]);
        }
        blk0++;
        prev_vs = vs;
      }
      // ---- PV1_{n-1}
      if (ok && two) {
        if (n == 1 && units1 > 0) ok = warp_wait(&bars->o_free[1], (units1 - 1) & 1, bars);
        if (ok) ok = warp_wait(&bars->p_full[1], blk1 & 1, bars);
        if (ok && lane == 0) {
          tc_fence_after_sync();
          issue_pv<kDt>(tmem + 384, tmem + 128, v_lo0 + prev_vs * kStageLo, hi, n - 1 > 0);
          tc_commit(&bars->o_final[1]);
          tc_commit(&bars->kv_empty[prev_vs]);
        }
        blk1++;
      }
    }
    units0++;
    if (two || halves) units1++;
  }
  // all MMAs issued by this thread complete before TMEM is released
  if (lane == 0) {
    tc_commit(&bars->drain);
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(&bars->drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
    }
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// softmax of a narrow tile (at most kNarrowRows live rows: decode with
// G <= 8).  The live rows sit in TMEM lanes 0..7, all read by the first warp
// of the warpgroup, which in the row-per-thread layout would spend 32 lanes
// of exp2 per live row.  Instead that warp moves the 8 rows of S through
// shared memory (the second Q slot, unused when every Q block is one tile)
// so that each lane takes 32 keys of one row: lane = 4 * row + segment.  Row
// maxima and sums reduce over the 4 lanes of a row; P goes back through
// shared memory to the row's own lane for the TMEM store.  Lanes 8..127 of
// S, P and O are padding rows that no output reads (their P is zero).  The
// other three warps of the warpgroup only keep the barrier counts.
// ---------------------------------------------------------------------------
// softmaxPrecision 1 (GBSA article, "Softmax precision": the softmax in half
// precision, the rescale in fp32): 32 scores s (fp32) of one row to their
// weights P = 2^(s * scale_log2 - m).  The exponent x is formed in fp32 (one
// f32x2 FMA per pair), rounded to an f16 pair, and one ex2.approx.f16x2 gives
// both weights in f16 -- half the MUFU operations of the fp32 path.  The f16
// weights are P itself for fp16 (ph), are rounded to bf16 for bf16 and cast
// to E4M3 for E4M3 (pk); the row sum adds the f16 weights widened exactly to
// fp32 (sp2, two lanes), so it sums the weights the P.V product uses.  The
// running max and the O rescale stay fp32.
template <int kDt, typename S>
__device__ __forceinline__ void exp2_half_chunk(const S (&sv)[32], uint64_t sc2, uint64_t nm2,
                                                uint32_t (&ph)[16],
                                                uint32_t (&pk)[kDt == kDtE4m3 ? 8 : 16],
                                                uint64_t& sp2) {
#pragma unroll
  for (int i = 0; i < 16; i++) {
    float x0, x1;
    f2_unpack(f2_fma(f2_pack(as_float(sv[2 * i]), as_float(sv[2 * i + 1])), sc2, nm2), x0, x1);
    ph[i] = exp2_f16x2(pack_f16x2(x0, x1));
    float e0, e1;
    f16x2_to_f32(ph[i], e0, e1);
    sp2 = f2_add(sp2, f2_pack(e0, e1));
    if constexpr (kDt == kDtBf16) pk[i] = pack_bf16x2(e0, e1);
    if constexpr (kDt == kDtFp16) pk[i] = ph[i];
    if constexpr (kDt == kDtE4m3) {
      if (i & 1) pk[i >> 1] = pack_e4m3x4_f16(ph[i - 1], ph[i]);
    }
  }
}

constexpr int kNarrowRows = 8;
constexpr int kNarrowSStride = 148;  // floats per S row (spreads banks for both access patterns)
constexpr int kNarrowSSeg = 36;      // floats between the 32-key segments of a row
constexpr int kNarrowPStride = 68;   // words per P row
constexpr int kNarrowSBytes = kNarrowRows * kNarrowSStride * 4;
constexpr int kNarrowPBytes = kNarrowRows * kNarrowPStride * 4;
static_assert(2 * kNarrowSBytes <= kHalfBytes && 2 * kNarrowPBytes <= kHalfBytes,
              "the narrow scratch fits the second Q slot");
static_assert(3 * kNarrowSSeg + 32 <= kNarrowSStride, "the segments fit a row");

// One block of a narrow tile, run by the warpgroup's first warp.  m and l
// are this lane's row statistics (m the same in the row's 4 lanes, l the
// lane's partial sum).  ri, key_lo and key_hi describe row lane / 4.
template <int kDt, bool kHalfSm>
__device__ __forceinline__ void softmax_narrow_block(const FwdParams& p, uint32_t t_s, uint32_t t_o,
                                                     float* scr_s, uint32_t* scr_p, int32_t entry,
                                                     const RowInfo& ri, int32_t key_lo,
                                                     int32_t key_hi, float& m, float& l,
                                                     uint32_t lane) {
  const int nrow = (int)(lane >> 2), seg = (int)(lane & 3);
#pragma unroll
  for (int h = 0; h < 2; h++) {  // 64 columns at a time
    uint32_t r[2][32];
    tmem_ld_32x32(t_s + 64 * h, r[0]);
    tmem_ld_32x32(t_s + 64 * h + 32, r[1]);
    tmem_wait_ld(r[0]);
    reg_fence(r[1]);
    if (lane < (uint32_t)kNarrowRows) {
      float* dst = scr_s + lane * kNarrowSStride + 2 * h * kNarrowSSeg;
#pragma unroll
      for (int q = 0; q < 2; q++)
#pragma unroll
        for (int i = 0; i < 8; i++)
          *reinterpret_cast<uint4*>(dst + q * kNarrowSSeg + 4 * i) =
              make_uint4(r[q][4 * i], r[q][4 * i + 1], r[q][4 * i + 2], r[q][4 * i + 3]);
    }
  }
  __syncwarp();
  float sv[32];
  {
    const float* src = scr_s + nrow * kNarrowSStride + seg * kNarrowSSeg;
#pragma unroll
    for (int i = 0; i < 8; i++) {
      const float4 v = *reinterpret_cast<const float4*>(src + 4 * i);
      sv[4 * i] = v.x;
      sv[4 * i + 1] = v.y;
      sv[4 * i + 2] = v.z;
      sv[4 * i + 3] = v.w;
    }
  }
  // visible keys of this block for the row: [clo, chi] (as in the wide path)
  int32_t clo = 0, chi = kPage - 1;
  if (!ri.used) {
    clo = kPage;
    chi = -1;
  } else if (entry & kEntryMask) {
    const int32_t base = (entry & kEntryLbMask) * kPage;
    clo = key_lo == INT32_MIN ? 0 : max(key_lo - base, 0);
    chi = min(key_hi - base, kPage - 1);
  }
  const int32_t k0 = seg * 32;
  if (__any_sync(0xffffffffu, clo > k0 || chi < k0 + 31)) {
#pragma unroll
    for (int c = 0; c < 32; c++)
      if (k0 + c < clo || k0 + c > chi) sv[c] = -INFINITY;
  }
  float mp[4];
#pragma unroll
  for (int k = 0; k < 4; k++) mp[k] = sv[k];
#pragma unroll
  for (int c = 4; c < 32; c += 2) mp[(c >> 1) & 3] = max3f(mp[(c >> 1) & 3], sv[c], sv[c + 1]);
  float mx = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const float m_blk = mx * p.scale_log2;
  const float m_new = fmaxf(m, m_blk);
  const bool rescale =
      m_new != -INFINITY && (m == -INFINITY || m_new > m + rescale_threshold<kDt>());
  const bool fix_o = rescale && m != -INFINITY;
  const float factor = fix_o ? fast_exp2(m - m_new) : 1.f;
  if (rescale) {
    l *= factor;
    m = m_new;
  }
  const float neg_m = ((m == -INFINITY) ? 0.f : -m) + (kDt == kDtE4m3 ? 8.f : 0.f);
  // the lane's 32 keys of P into the row's P line
  constexpr int kPw = kDt == kDtE4m3 ? 8 : 16;  // words per 32 keys
  {
    uint32_t pk[kPw];
    if constexpr (kHalfSm) {
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(neg_m, neg_m);
      uint64_t sp2 = 0ull;
      uint32_t ph[16];
      exp2_half_chunk<kDt>(sv, sc2, nm2, ph, pk, sp2);
      float s0, s1;
      f2_unpack(sp2, s0, s1);
      l += s0 + s1;
    } else {
      float pf[32];
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        pf[c] = fast_exp2(fmaf(sv[c], p.scale_log2, neg_m));
        pf[c + 1] = fast_exp2(fmaf(sv[c + 1], p.scale_log2, neg_m));
        s0 += pf[c];
        s1 += pf[c + 1];
      }
      l += s0 + s1;
      if constexpr (kDt == kDtE4m3) {
#pragma unroll
        for (int i = 0; i < 8; i++)
          pk[i] = pack_e4m3x4(pf[4 * i], pf[4 * i + 1], pf[4 * i + 2], pf[4 * i + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 16; i++) pk[i] = pack_x2<kDt == kDtFp16>(pf[2 * i], pf[2 * i + 1]);
      }
    }
    uint32_t* dst = scr_p + nrow * kNarrowPStride + seg * kPw;
#pragma unroll
    for (int i = 0; i < kPw / 4; i++)
      *reinterpret_cast<uint4*>(dst + 4 * i) =
          make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
  }
  __syncwarp();
  // lane r < 8 stores row r's P (4 * kPw words) into its TMEM lane; the
  // padding lanes store zeros
  {
    const bool own = lane < (uint32_t)kNarrowRows;
    const uint32_t* src = scr_p + (lane & (kNarrowRows - 1)) * kNarrowPStride;
#pragma unroll
    for (int q = 0; q < 4; q++) {
      uint32_t w[kPw];
#pragma unroll
      for (int i = 0; i < kPw / 4; i++) {
        const uint4 v = own ? *reinterpret_cast<const uint4*>(src + q * kPw + 4 * i)
                            : make_uint4(0u, 0u, 0u, 0u);
        w[4 * i] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
      }
      if constexpr (kDt == kDtE4m3)
        tmem_st_32x8(t_s + 8 * q, w);
      else
        tmem_st_32x16(t_s + 16 * q, w);
    }
  }
  // O of the live rows to the new reference max (row r's factor is held by
  // lanes 4r..4r+3)
  const int src_lane = (int)(lane & (kNarrowRows - 1)) * 4;
  const float f_own = __shfl_sync(0xffffffffu, factor, src_lane);
  const bool fix_own =
      __shfl_sync(0xffffffffu, fix_o ? 1 : 0, src_lane) != 0 && lane < (uint32_t)kNarrowRows;
  if (__any_sync(0xffffffffu, fix_own)) {
    const float f = fix_own ? f_own : 1.f;
#pragma unroll 1
    for (int c = 0; c < 4; c++) {
      uint32_t o[32];
      tmem_ld_32x32(t_o + 32 * c, o);
      tmem_wait_ld(o);
#pragma unroll
      for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
      tmem_st_32x32(t_o + 32 * c, o);
    }
  }
}

// ---------------------------------------------------------------------------
// softmax (one warpgroup per tile slot; thread = tile row = TMEM lane)
// ---------------------------------------------------------------------------
// The kernel's dynamic shared memory (every extern __shared__ array starts at
// the same address): offsets from it are constants, with no register.
__device__ __forceinline__ uint8_t* dyn_smem() {
  extern __shared__ __align__(1024) uint8_t dsm[];
  return dsm;
}

template <bool kHalves, int kDt, bool kHalfSm>
__device__ void run_softmax(const FwdParams& p, Bars* bars, uint32_t tmem, int slot,
                            int64_t off_list) {
  const int row = threadIdx.x & 127;
  const uint32_t lane_sel = (uint32_t)(threadIdx.x & 96) << 16;  // warp's 32-lane quarter
  const uint32_t t_s = tmem + 128 * slot + lane_sel;
  const uint32_t t_o = tmem + 256 + 128 * slot + lane_sel;
  // narrow tiles (the one-tile instantiation only: the second Q slot is free)
  const bool narrow = kHalves && p.tile_tokens * p.G <= kNarrowRows;
  uint32_t blk = 0, units = 0;
  UnitRec ur;
  for (UnitCursor cur; cur.next(bars, ur);) {
    const Unit x = decode_unit<kHalves>(ur, p.N2);
    const int32_t nblk = x.j1 - x.j0;
    if ((slot >= x.nt && !x.halves) || nblk <= 0) continue;
    // a unit in halves: both slots hold the rows of its one tile, slot s
    // takes blocks s, s + 2, ...  (narrow: this lane works on row lane / 4)
    const bool narrow_lead = narrow && (threadIdx.x & 96) == 0;
    const RowInfo ri = row_info(p, x, x.halves ? 0 : slot, narrow_lead ? (row >> 2) : row);
    const int32_t jb0 = x.halves ? slot : 0, jstep = x.halves ? 2 : 1;
    const int32_t key_hi = min(ri.pos, x.ku - 1);
    const int32_t key_lo = p.win_left >= 0 ? ri.pos - p.win_left : INT32_MIN;
    const int32_t* list = p.meta + off_list + (int64_t)x.item * p.top_k + x.j0;
    float m = -INFINITY, l = 0.f;
    if (kHalves && narrow) {
      for (int32_t jb = jb0; jb < nblk; jb += jstep) {
        const int32_t entry = list[jb];
        if (!wait_bar(&bars->s_full[slot], blk & 1, bars)) return;
        if (narrow_lead) {
          tc_fence_after_sync();
          float* scr_s =
              reinterpret_cast<float*>(dyn_smem() + kSmemQ + kTileBytes + slot * kNarrowSBytes);
          uint32_t* scr_p = reinterpret_cast<uint32_t*>(dyn_smem() + kSmemQ + kTileBytes +
                                                        kHalfBytes + slot * kNarrowPBytes);
          softmax_narrow_block<kDt, kHalfSm>(p, t_s, t_o, scr_s, scr_p, entry, ri, key_lo,
                                             key_hi, m, l, lane_id());
          tmem_wait_st();
          tc_fence_before_sync();
        }
        mbar_arrive(&bars->p_full[slot]);
        blk++;
      }
    } else {
      for (int32_t jb = jb0; jb < nblk; jb += jstep) {
        const int32_t entry = list[jb];
        if (!wait_bar(&bars->s_full[slot], blk & 1, bars)) return;
        tc_fence_after_sync();
        uint32_t r[4][32];
        tmem_ld_32x32(t_s + 0, r[0]);
        tmem_ld_32x32(t_s + 32, r[1]);
        tmem_ld_32x32(t_s + 64, r[2]);
        tmem_ld_32x32(t_s + 96, r[3]);
        tmem_wait_ld(r[0]);
        reg_fence(r[1]);
        reg_fence(r[2]);
        reg_fence(r[3]);
        // visible key columns of this block for this row: [clo, chi].  A row
        // whose output is never written (padding rows of a tile, rows past
        // seqused_q) is left unmasked: its softmax only feeds its own row of
        // P and O, which no output reads, and it never rescales O (below).
        // The element mask runs per 32-column chunk, only in warps where some
        // row needs it there.
        int32_t clo = 0, chi = kPage - 1;
        if (ri.used && (entry & kEntryMask)) {
          const int32_t base = (entry & kEntryLbMask) * kPage;
          clo = key_lo == INT32_MIN ? 0 : max(key_lo - base, 0);
          chi = min(key_hi - base, kPage - 1);
        }
        if (__any_sync(0xffffffffu, clo > 0 || chi < kPage - 1)) {
  #pragma unroll
          for (int q = 0; q < 4; q++) {
            if (__any_sync(0xffffffffu, clo > 32 * q || chi < 32 * q + 31)) {
  #pragma unroll
              for (int c = 0; c < 32; c++)
                if (32 * q + c < clo || 32 * q + c > chi) r[q][c] = __float_as_uint(-INFINITY);
            }
          }
        }
        // row max: eight independent partial maxima, then a tree
        float mp[8];
  #pragma unroll
        for (int k = 0; k < 8; k++) mp[k] = __uint_as_float(r[0][k]);
  #pragma unroll
        for (int c = 8; c < 128; c += 2)
          mp[(c >> 1) & 7] = max3f(mp[(c >> 1) & 7], __uint_as_float(r[c >> 5][c & 31]),
                                   __uint_as_float(r[c >> 5][(c + 1) & 31]));
        const float mx = max3f(max3f(mp[0], mp[1], mp[2]), max3f(mp[3], mp[4], mp[5]),
                               fmaxf(mp[6], mp[7]));
        const float m_blk = mx * p.scale_log2;
        const float m_new = fmaxf(m, m_blk);
        // lazy rescale: keep the old reference max unless it grew past the
        // threshold (rows whose output is never written keep m = -inf)
        const bool rescale = ri.used && m_new != -INFINITY &&
                             (m == -INFINITY || m_new > m + rescale_threshold<kDt>());
        const bool fix_o = rescale && m != -INFINITY;
        const float factor = fix_o ? fast_exp2(m - m_new) : 1.f;
        if (rescale) {
          l *= factor;
          m = m_new;
        }
        // E4M3 P carries a factor 2^8 (the row sum l too; the statistics
        // handed on below take it out of m)
        const float neg_m = ((m == -INFINITY) ? 0.f : -m) + (kDt == kDtE4m3 ? 8.f : 0.f);
        // scores pairwise: x = s * scale_log2 - m as one f32x2 FMA, P = 2^x,
        // the row sum in two packed partial sums (four independent lanes)
        const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nm2 = f2_pack(neg_m, neg_m);
        uint64_t sp2[2] = {0ull, 0ull};
  #pragma unroll
        for (int q = 0; q < 4; q++) {
          if constexpr (kHalfSm) {
            uint32_t ph[16];
            uint32_t pk[kDt == kDtE4m3 ? 8 : 16];
            exp2_half_chunk<kDt>(r[q], sc2, nm2, ph, pk, sp2[q & 1]);
            if constexpr (kDt == kDtE4m3)
              tmem_st_32x8(t_s + 8 * q, pk);
            else
              tmem_st_32x16(t_s + 16 * q, pk);
          } else {
            float pf[32];
  #pragma unroll
            for (int i = 0; i < 16; i++) {
              // masked scores are -inf and ex2(-inf) = +0
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(r[q][2 * i]),
                                       __uint_as_float(r[q][2 * i + 1])),
                               sc2, nm2),
                        x0, x1);
              pf[2 * i] = fast_exp2(x0);
              pf[2 * i + 1] = fast_exp2(x1);
              sp2[i & 1] = f2_add(sp2[i & 1], f2_pack(pf[2 * i], pf[2 * i + 1]));
            }
            if constexpr (kDt == kDtE4m3) {
              // four E4M3 weights per TMEM column: 32 keys in 8 columns
              uint32_t pk[8];
  #pragma unroll
              for (int i = 0; i < 8; i++)
                pk[i] = pack_e4m3x4(pf[4 * i], pf[4 * i + 1], pf[4 * i + 2], pf[4 * i + 3]);
              tmem_st_32x8(t_s + 8 * q, pk);
            } else {
              uint32_t pk[16];
  #pragma unroll
              for (int i = 0; i < 16; i++)
                pk[i] = pack_x2<kDt == kDtFp16>(pf[2 * i], pf[2 * i + 1]);
              tmem_st_32x16(t_s + 16 * q, pk);
            }
          }
        }
        float s0, s1, s2, s3;
        f2_unpack(sp2[0], s0, s1);
        f2_unpack(sp2[1], s2, s3);
        l += (s0 + s1) + (s2 + s3);
        if (__any_sync(0xffffffffu, fix_o)) {
          // O holds the earlier blocks (their PV completed before this S was
          // committed); bring it to the new reference max.
  #pragma unroll 1
          for (int c = 0; c < 4; c++) {
            uint32_t o[32];
            tmem_ld_32x32(t_o + 32 * c, o);
            tmem_wait_ld(o);
  #pragma unroll
            for (int i = 0; i < 32; i++) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
            tmem_st_32x32(t_o + 32 * c, o);
          }
        }
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&bars->p_full[slot]);
        blk++;
      }
    }
    if (kHalves && narrow) {
      // row sums over the 4 lanes of a row, then lane r takes row r's
      // statistics (rows past the live ones, and the other warps: none)
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      const uint32_t lane = lane_id();
      const int src_lane = (int)(lane & (kNarrowRows - 1)) * 4;
      const float m_r = __shfl_sync(0xffffffffu, m, src_lane);
      const float l_r = __shfl_sync(0xffffffffu, l, src_lane);
      const bool live = (threadIdx.x & 96) == 0 && lane < (uint32_t)kNarrowRows;
      m = live ? m_r : -INFINITY;
      l = live ? l_r : 0.f;
    }
    // hand the row statistics of this unit to the epilogue warpgroup
    if (units > 0 && !wait_bar(&bars->stats_free[slot], (units - 1) & 1, bars)) return;
    // (E4M3: P and l carry 2^8, so the reference max handed on is m - 8)
    bars->stats[slot][row] = make_float2(kDt == kDtE4m3 && m != -INFINITY ? m - 8.f : m, l);
    mbar_arrive(&bars->stats_full[slot]);
    units++;
  }
}

// ---------------------------------------------------------------------------
// epilogue (one warpgroup; thread = tile row = TMEM lane, both tile slots)
// ---------------------------------------------------------------------------
// E4M3 V carries a per-tensor dequantization scale, applied with 1 / l (the
// split-KV partials too: the merge is linear in them).
template <int kDt>
__device__ __forceinline__ float out_numerator(const FwdParams& p) {
  return kDt == kDtE4m3 ? p.out_scale : 1.f;
}

template <bool kHalves, int kDt>
__device__ void run_epilogue(const FwdParams& p, Bars* bars, uint32_t tmem) {
  const int row = threadIdx.x & 127;
  const uint32_t lane_sel = (uint32_t)(threadIdx.x & 96) << 16;
  const int rows_in_tile = p.tile_tokens * p.G;
  uint32_t units_stats[2] = {0, 0}, units_final[2] = {0, 0};
  int32_t bad = 0;
  bool ok = true;
  UnitRec ur;
  for (UnitCursor cur; ok && cur.next(bars, ur);) {
    const Unit x = decode_unit<kHalves>(ur, p.N2);
    const int32_t nblk = x.j1 - x.j0;
    if (x.halves) {
      // two partial softmaxes over the even and odd blocks of one tile:
      // O = (O0 2^(m0-M) + O1 2^(m1-M)) / (l0 2^(m0-M) + l1 2^(m1-M)), M = max
      const RowInfo ri = row_info(p, x, 0, row);
      float2 st[2];
      for (int s = 0; s < 2 && ok; s++) {
        if (!(ok = wait_bar(&bars->stats_full[s], units_stats[s] & 1, bars))) break;
        st[s] = bars->stats[s][row];
        mbar_arrive(&bars->stats_free[s]);
        units_stats[s]++;
      }
      for (int s = 0; s < 2 && ok; s++) {
        if (!(ok = wait_bar(&bars->o_final[s], units_final[s] & 1, bars))) break;
        units_final[s]++;
      }
      if (!ok) break;
      tc_fence_after_sync();
      const float mm = fmaxf(st[0].x, st[1].x);
      const float w0 = st[0].y > 0.f ? fast_exp2(st[0].x - mm) : 0.f;
      const float w1 = st[1].y > 0.f ? fast_exp2(st[1].x - mm) : 0.f;
      const float l = st[0].y * w0 + st[1].y * w1;
      const bool has = ri.used && l > 0.f;
      const float inv_l = has ? out_numerator<kDt>(p) / l : 0.f;
      const float a0 = w0 * inv_l, a1 = w1 * inv_l;
      const float lse = has ? (mm + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const bool write_row = ri.store && ri.tok < p.T;
      if (ri.store && ri.tok >= p.T) bad |= kDevBadSeqlen;
      const uint32_t t_o0 = tmem + 256 + lane_sel, t_o1 = tmem + 384 + lane_sel;
      if (x.slot < 0) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((int64_t)ri.tok * p.N1 + ri.h) * kHeadDim);
#pragma unroll 1
        for (int c = 0; c < 16; c++) {
          uint32_t o0[8], o1[8];
          tmem_ld_2x32x8_wait(t_o0 + 8 * c, t_o1 + 8 * c, o0, o1);
          uint32_t pk[4];
#pragma unroll
          for (int i = 0; i < 4; i++)
            pk[i] = has ? pack_x2<kDt == kDtFp16>(
                              __uint_as_float(o0[2 * i]) * a0 + __uint_as_float(o1[2 * i]) * a1,
                              __uint_as_float(o0[2 * i + 1]) * a0 + __uint_as_float(o1[2 * i + 1]) * a1)
                        : 0u;
          if (write_row) dst[c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        if (write_row && p.return_lse) p.lse[(int64_t)ri.tok * p.N1 + ri.h] = lse;
      } else {
        const int64_t wrow = (int64_t)x.slot * p.rows_per_unit + row;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + wrow * kHeadDim);
#pragma unroll 1
        for (int c = 0; c < 16; c++) {
          uint32_t o0[8], o1[8];
          tmem_ld_2x32x8_wait(t_o0 + 8 * c, t_o1 + 8 * c, o0, o1);
          if (row < rows_in_tile) {
#pragma unroll
            for (int i = 0; i < 2; i++) {
              float v[4];
#pragma unroll
              for (int e = 0; e < 4; e++)
                v[e] = has ? __uint_as_float(o0[4 * i + e]) * a0 + __uint_as_float(o1[4 * i + e]) * a1
                           : 0.f;
              dst[2 * c + i] = make_float4(v[0], v[1], v[2], v[3]);
            }
          }
        }
        if (row < rows_in_tile) p.ws_lse[wrow] = lse;
      }
      tc_fence_before_sync();
      mbar_arrive(&bars->o_free[0]);
      mbar_arrive(&bars->o_free[1]);
      continue;
    }
    for (int slot = 0; slot < x.nt && ok; slot++) {
      const RowInfo ri = row_info(p, x, slot, row);
      const uint32_t t_o = tmem + 256 + 128 * slot + lane_sel;
      float m = -INFINITY, l = 0.f;
      if (nblk > 0) {
        if (!(ok = wait_bar(&bars->stats_full[slot], units_stats[slot] & 1, bars))) break;
        const float2 st = bars->stats[slot][row];
        m = st.x;
        l = st.y;
        mbar_arrive(&bars->stats_free[slot]);
        units_stats[slot]++;
        if (!(ok = wait_bar(&bars->o_final[slot], units_final[slot] & 1, bars))) break;
        units_final[slot]++;
        tc_fence_after_sync();
      }
      const bool has = nblk > 0 && ri.used && l > 0.f;
      const float inv_l = has ? out_numerator<kDt>(p) / l : 0.f;
      const float lse = has ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      const bool write_row = ri.store && ri.tok < p.T;
      if (ri.store && ri.tok >= p.T) bad |= kDevBadSeqlen;
      if (x.slot < 0) {
        uint4* dst = reinterpret_cast<uint4*>(p.out + ((int64_t)ri.tok * p.N1 + ri.h) * kHeadDim);
#pragma unroll 1
        for (int c = 0; c < 8; c++) {
          uint32_t o[16];
          if (nblk > 0) tmem_ld_32x16_wait(t_o + 16 * c, o);
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; i++)
            pk[i] = has ? pack_x2<kDt == kDtFp16>(__uint_as_float(o[2 * i]) * inv_l,
                                      __uint_as_float(o[2 * i + 1]) * inv_l)
                        : 0u;
          if (write_row) {
            dst[2 * c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            dst[2 * c + 1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
        if (write_row && p.return_lse) p.lse[(int64_t)ri.tok * p.N1 + ri.h] = lse;
      } else {
        const int64_t wrow = (int64_t)x.slot * p.rows_per_unit + slot * rows_in_tile + row;
        float4* dst = reinterpret_cast<float4*>(p.ws_o + wrow * kHeadDim);
#pragma unroll 1
        for (int c = 0; c < 8; c++) {
          uint32_t o[16];
          if (nblk > 0) tmem_ld_32x16_wait(t_o + 16 * c, o);
          if (row < rows_in_tile) {
#pragma unroll
            for (int i = 0; i < 4; i++)
              dst[4 * c + i] = has ? make_float4(__uint_as_float(o[4 * i]) * inv_l,
                                                 __uint_as_float(o[4 * i + 1]) * inv_l,
                                                 __uint_as_float(o[4 * i + 2]) * inv_l,
                                                 __uint_as_float(o[4 * i + 3]) * inv_l)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        if (row < rows_in_tile) p.ws_lse[wrow] = lse;
      }
      tc_fence_before_sync();
      mbar_arrive(&bars->o_free[slot]);
    }
  }
  if (bad && p.dev_status) atomicOr(p.dev_status, bad);
}

template <bool kHalves, int kDt, bool kHalfSm>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_v, const FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  allow_dependents();
  grid_dependency_wait();  // the work list (and, before it, q, k and v)

  // the work list must have been built for this problem, and the swizzled
  // tiles need a 1 KiB aligned shared-memory window
  const int32_t* meta = p.meta;
  const bool match = (uint32_t)meta[H_MAGIC] == kMagic && meta[H_VERSION] == kFormatVersion &&
                     (uint32_t)meta[H_SIGNATURE] == p.signature;
  if (!match || (smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && p.dev_status)
      atomicOr(p.dev_status, match ? kDevTimeout : kDevMetaMismatch);
    return;
  }
  const int32_t n_units = meta[H_NUNITS];
  const int64_t off_unit = meta[H_OFF_UNIT], off_item = meta[H_OFF_ITEM], off_list = meta[H_OFF_LIST];
  if ((int32_t)blockIdx.x >= n_units) return;  // no work for this CTA (uniform)

  Bars* bars = reinterpret_cast<Bars*>(smem + kSmemBars);
  if (threadIdx.x == 0) {
    for (uint32_t i = 0; i < kUnitQ; i++) {
      mbar_init(&bars->uq_full[i], 1);
      mbar_init(&bars->uq_empty[i], kUnitReaders);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->q_empty[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_final[i], 1);
      mbar_init(&bars->o_free[i], 128);
      mbar_init(&bars->stats_full[i], 128);
      mbar_init(&bars->stats_free[i], 128);
    }
    for (int i = 0; i < kMaxStages; i++) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->wait_limit_ns = p.wait_limit_ns;
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = bars->tmem_base;

  if (warp < 8) {
    setmaxnreg_inc<regs_softmax<kHalves>()>();
    run_softmax<kHalves, kDt, kHalfSm>(p, bars, tmem, warp >> 2, off_list);
  } else if (warp < 12) {
    setmaxnreg_dec<kRegsEpilogue>();
    run_epilogue<kHalves, kDt>(p, bars, tmem);
  } else {
    setmaxnreg_dec<regs_control<kHalves>()>();
    if (warp == kWarpMma) {
      run_mma<kHalves, kDt>(p, smem, bars, tmem, off_list);
    } else if (warp == kWarpProducer) {
      if (lane_id() == 0) {
        tma_prefetch_map(&map_q);
        tma_prefetch_map(&map_k);
        tma_prefetch_map(&map_v);
      }
      run_producer<kHalves, kDt>(p, &map_q, &map_k, &map_v, smem, bars, n_units, off_unit, off_item, off_list);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0 && bars->abort && p.dev_status) atomicOr(p.dev_status, kDevTimeout);
  if (warp == kWarpMma) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// split-KV combine: one CTA per split (item, tile pair); a warp per row
// ---------------------------------------------------------------------------
struct CombineParams {
  const int32_t* meta;
  const float* ws_o;
  const float* ws_lse;
  uint16_t* out;  // fp16 for fp16 inputs, else bf16
  float* lse;
  int32_t* dev_status;
  uint32_t signature;
  int32_t N1, N2, G, T, tile_tokens, rows_per_unit, return_lse, fp16;
};

__global__ void __launch_bounds__(256) combine_kernel(const CombineParams p) {
  grid_dependency_wait();  // the forward's partials
  const int32_t* meta = p.meta;
  if ((uint32_t)meta[H_MAGIC] != kMagic || (uint32_t)meta[H_SIGNATURE] != p.signature) return;
  const int32_t n_comb = meta[H_NCOMB];
  if ((int32_t)blockIdx.x >= n_comb) return;
  const int4 rec = *reinterpret_cast<const int4*>(meta + meta[H_OFF_COMB] + 4 * (int64_t)blockIdx.x);
  const int32_t item = rec.x, tp = rec.y, first = rec.z, k = rec.w;
  const int32_t* it = meta + meta[H_OFF_ITEM] + 8 * (int64_t)item;
  const int32_t n_tiles = it[2], tok_begin = it[3], n_store = it[4];
  const int32_t kvh = item % p.N2;
  const int rows_in_tile = p.tile_tokens * p.G;
  const int lane = threadIdx.x & 31;
  const int nt = min(2, n_tiles - 2 * tp);
  for (int rr = threadIdx.x >> 5; rr < nt * rows_in_tile; rr += blockDim.x >> 5) {
    const int s = rr / rows_in_tile, row = rr - s * rows_in_tile;
    const int32_t tok_off = (2 * tp + s) * p.tile_tokens + row / p.G;
    if (tok_off >= n_store) continue;
    const int32_t tok = tok_begin + tok_off;
    if (tok >= p.T) continue;
    const int32_t h = kvh * p.G + row % p.G;
    const int64_t wrow0 = (int64_t)first * p.rows_per_unit + rr;
    float mx = -INFINITY;
    for (int j = 0; j < k; j++) mx = fmaxf(mx, p.ws_lse[wrow0 + (int64_t)j * p.rows_per_unit]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (mx != -INFINITY) {
      for (int j = 0; j < k; j++) {
        const int64_t wrow = wrow0 + (int64_t)j * p.rows_per_unit;
        const float lj = p.ws_lse[wrow];
        const float w = lj == -INFINITY ? 0.f : expf(lj - mx);
        wsum += w;
        const float4 o = reinterpret_cast<const float4*>(p.ws_o + wrow * kHeadDim)[lane];
        acc.x += w * o.x;
        acc.y += w * o.y;
        acc.z += w * o.z;
        acc.w += w * o.w;
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint2 pk;
    pk.x = p.fp16 ? pack_f16x2(acc.x * inv, acc.y * inv) : pack_bf16x2(acc.x * inv, acc.y * inv);
    pk.y = p.fp16 ? pack_f16x2(acc.z * inv, acc.w * inv) : pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(p.out + ((int64_t)tok * p.N1 + h) * kHeadDim)[lane] = pk;
    if (lane == 0 && p.return_lse)
      p.lse[(int64_t)tok * p.N1 + h] = wsum > 0.f ? mx + logf(wsum) : -INFINITY;
  }
}

}  // namespace

size_t forward_smem_bytes() { return kSmemBytes; }

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
                           uint64_t wait_limit_ns, cudaStream_t stream) {
  using Kernel = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const FwdParams);
  // [element type][softmax precision][one_tile_blocks]
  static const Kernel kernels[3][2][2] = {
      {{fwd_kernel<false, kDtBf16, false>, fwd_kernel<true, kDtBf16, false>},
       {fwd_kernel<false, kDtBf16, true>, fwd_kernel<true, kDtBf16, true>}},
      {{fwd_kernel<false, kDtFp16, false>, fwd_kernel<true, kDtFp16, false>},
       {fwd_kernel<false, kDtFp16, true>, fwd_kernel<true, kDtFp16, true>}},
      {{fwd_kernel<false, kDtE4m3, false>, fwd_kernel<true, kDtE4m3, false>},
       {fwd_kernel<false, kDtE4m3, true>, fwd_kernel<true, kDtE4m3, true>}}};
  if (dtype < 0 || dtype > 2) return cudaErrorInvalidValue;
  static int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    // The register re-split is only safe if the kernel launches with exactly
    // the registers the split was computed for.
    for (int i = 0; i < 12; i++) {
      const void* fn = reinterpret_cast<const void*>(kernels[i / 4][(i / 2) % 2][i % 2]);
      cudaFuncAttributes attr;
      e = cudaFuncGetAttributes(&attr, fn);
      if (e != cudaSuccess) return e;
      if (attr.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
      if (e != cudaSuccess) return e;
    }
    configured_device = dev;
  }
  FwdParams p;
  p.meta = meta;
  p.work = meta + H_UNIT_NEXT;
  p.block_table = block_table;
  p.cu_kv = cu_seqlens_kv;
  p.out = static_cast<uint16_t*>(out);
  p.lse = lse;
  p.ws_o = ws_o;
  p.ws_lse = ws_lse;
  p.dev_status = dev_status;
  p.signature = signature;
  p.N1 = N1;
  p.N2 = N2;
  p.G = N1 / N2;
  p.T = T;
  p.top_k = top_k;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.tile_tokens = tile_tokens;
  p.rows_per_unit = rows_per_unit;
  p.win_left = win_left;
  p.return_lse = return_lse;
  p.scale_log2 = scale_log2;
  p.out_scale = out_scale;
  p.wait_limit_ns = wait_limit_ns;
  // every Q block in one tile (decode-like): the instantiation with units in
  // halves; the element type picks the MMA kind, P's format and the output type
  {
    NvtxRange range("gbsa_forward");
    e = launch_dependent(kernels[dtype][half_softmax ? 1 : 0][one_tile_blocks ? 1 : 0],
                         dim3(num_ctas),
                         dim3(kThreads), kSmemBytes, stream, map_q, map_k, map_v, p);
  }
  if (e != cudaSuccess || comb_cap <= 0) return e;
  CombineParams c;
  c.meta = meta;
  c.ws_o = ws_o;
  c.ws_lse = ws_lse;
  c.out = p.out;
  c.lse = lse;
  c.dev_status = dev_status;
  c.signature = signature;
  c.N1 = N1;
  c.N2 = N2;
  c.G = p.G;
  c.T = T;
  c.tile_tokens = tile_tokens;
  c.rows_per_unit = rows_per_unit;
  c.return_lse = return_lse;
  c.fp16 = dtype == kDtFp16 ? 1 : 0;
  NvtxRange range("gbsa_combine");
  return launch_dependent(combine_kernel, dim3((unsigned)comb_cap), dim3(256), 0, stream, c);
}

}  // namespace gbsa
