// gbsa_internal.cuh -- layout of the metadata buffer (format 1) and the
// launch geometry shared by the host library and the GBSA kernels.
//
// Metadata format 1, in int32 words (the GBSA article, cf-1.com/news/4865651,
// "two-phase call", gives the metadata its role -- the load-balanced task
// split computed before the main operator -- but not its content):
//
//   header      kHeaderWords words, fields HdrField below
//   seq table   B rows x 8:        qs, qu, ku, n_qblocks, qblock_base, tok_begin, 0, 0
//   item table  n_items rows x 8:  b, n_live, n_tiles, tok_begin, n_store, n_used, pos0, ku
//               item i = qb * N2 + kvh (Q-block major, then KV head)
//   live lists  n_items rows x top_k: lb | kEntryMask | kEntryPartial, list
//               order kept, dead entries dropped, the rest of each row 0
//   units       unit_cap rows x 4: item, tp, j0 | j1 << 16, slot (-1 = whole)
//               longest first (stable), n_units rows defined
//   combine     comb_cap rows x 4: item, tp, first_slot, n_pieces
//
// Tiling: G = N1/N2 query heads of one KV head and tile_tokens =
// min(128 / G, block_x) consecutive tokens form one 128-row MMA tile
// (row r <-> token r / G, head r % G, "packed GQA": the heads of a group
// share every K/V tile, GBSA article "Parameters" / is_packed_gqa).  A unit
// is a pair of tiles (tp) of one item.  An entry is live when some used row
// of the item sees some key of its block; kEntryMask marks blocks where some
// (row, key) pair is hidden, kEntryPartial a last page with keys >= seqused_kv.
#pragma once

#include <stdint.h>
#ifdef __CUDACC__
#include <cuda_runtime.h>
#endif
#include <nvtx3/nvToolsExt.h>

namespace gbsa {

// An NVTX range in the "gbsa" domain around the host code that enqueues one
// launch group (metadata, forward, combine), so that a profiler's timeline
// names them.  Header-only NVTX: without a tool attached it costs a branch.
class NvtxRange {
 public:
  explicit NvtxRange(const char* name) {
    static const nvtxDomainHandle_t domain = nvtxDomainCreateA("gbsa");
    domain_ = domain;
    nvtxEventAttributes_t a = {};
    a.version = NVTX_VERSION;
    a.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
    a.messageType = NVTX_MESSAGE_TYPE_ASCII;
    a.message.ascii = name;
    nvtxDomainRangePushEx(domain_, &a);
  }
  ~NvtxRange() { nvtxDomainRangePop(domain_); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;

 private:
  nvtxDomainHandle_t domain_;
};

constexpr int kPage = 128;        // keys per KV block = page size (blockShapeY)
constexpr int kHeadDim = 128;     // D
constexpr int kTileRows = 128;    // MMA M
constexpr int kHeaderWords = 32;
constexpr uint32_t kMagic = 0x41534247u;
constexpr int kFormatVersion = 1;
constexpr int32_t kEntryLbMask = 0x00FFFFFF;
constexpr int32_t kEntryMask = 1 << 24;
constexpr int32_t kEntryPartial = 1 << 25;
constexpr int kMinSplitLen = 8;
constexpr int kMaxTopK = 256;

enum HdrField : int {
  H_MAGIC = 0, H_VERSION, H_SIGNATURE, H_B, H_NITEMS, H_TILE_TOKENS, H_TILES_MAX, H_NUM_CTAS,
  H_UNIT_CAP, H_SLOT_CAP, H_COMB_CAP, H_NUNITS, H_NSLOTS, H_NCOMB, H_SPLIT_LEN, H_STATUS,
  H_COST_LO, H_COST_HI, H_OFF_SEQ, H_OFF_ITEM, H_OFF_LIST, H_OFF_UNIT, H_OFF_COMB, H_TOTAL,
  H_ROWS_PER_UNIT, H_G,
  // Work counters of the forward (zero when the metadata is built; each
  // forward launch fetches units through H_UNIT_NEXT and counts finished CTAs
  // in H_CTAS_DONE, and its last CTA puts both back to zero).
  H_UNIT_NEXT, H_CTAS_DONE
};

// Device-status bits (mirrors GBSA_DEV_* in include/gbsa.h).
constexpr int32_t kDevBadSeqlen = 0x01;
constexpr int32_t kDevBadBlockIdx = 0x02;
constexpr int32_t kDevBadCount = 0x04;
constexpr int32_t kDevBadPage = 0x08;
constexpr int32_t kDevMetaMismatch = 0x10;
constexpr int32_t kDevTimeout = 0x20;
constexpr int32_t kDevCapacity = 0x40;

struct Geometry {
  int32_t G, tile_tokens, tiles_max, n_items;
  int64_t unit_cap, slot_cap, comb_cap;
  int64_t off_seq, off_item, off_list, off_unit, off_comb, total_words;
  int32_t rows_per_unit;
};

// Host-known problem fields the kernels need (subset of gbsa_problem).
struct MetaParams {
  int32_t B, T, N1, N2, block_x, total_q_blocks, top_k, win_left, win_right, has_seqused_q;
  int32_t num_ctas, forced_split;
  uint32_t signature;
  Geometry geo;
  const int32_t* sparse_idx;
  const int32_t* sparse_count;
  const int64_t* cu_seqlens_q;
  const int32_t* seqused_q;
  const int32_t* seqused_kv;
  int32_t* meta;
  int32_t* dev_status;
};

#ifdef __CUDACC__
// Programmatic dependent launch.  Every kernel after the first of a call is
// launched with programmatic stream serialization: it may start while the
// kernel before it in the stream is still running, and waits in
// grid_dependency_wait() -- before it touches global memory -- until that
// kernel has completed and its writes are visible.  allow_dependents() lets
// the next kernel start early (it still waits for this one to complete).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}
#endif

}  // namespace gbsa
