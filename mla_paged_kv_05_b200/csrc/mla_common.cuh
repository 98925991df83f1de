// Shapes, workspace layout and kernel parameters shared by the MLA decode
// planner (K0), main kernel (K1) and split-combine kernel (K2).
//
// Absorbed MLA decode (evermx.com, "TokenSpeed: speed-of-light LLM inference
// engine for agentic workloads", section "Pluggable Kernel Registry": an MLA
// decode kernel under speculative decoding): one 576-wide latent row per token
// (512 compressed + 64 RoPE) shared by all heads, V = its first 512 columns,
// pages of 64 tokens reached through a block table (zubnet.ai "LightSeek
// TokenSpeed 580 TPS ... B200", second paragraph: KV pages and index
// indirection instead of copies).
#pragma once

#include <cstddef>
#include <cstdint>

namespace mla {

constexpr int kPage = 64;        // tokens per page = tokens per KV tile
constexpr int kDqk = 576;        // latent + rope width
constexpr int kDv = 512;         // value width (first 512 columns)
constexpr int kRowsPerTile = 128;  // partial-slot stride in rows (the largest tile height)
constexpr int kFp8PageBytes = kPage * kDqk + kPage * 4;  // codes + fp32 token scales

// Planner cost model, in units of one page of work per cluster.
constexpr int kSeqOverhead = 2;  // fixed cost of one (sequence, cluster) segment
constexpr int kMinPayload = 4;   // never cut work into pieces smaller than this

// Planner CTAs (besides the planning one) that range-check the block table.
constexpr int kMaxCheckCtas = 8;
constexpr int kCheckEntriesPerCta = 4096;

// Batches of at most this many sequences are planned by the decode kernel
// itself (each CTA derives the plan from the sequence lengths while it sets
// up, so it need not wait for the planner kernel), and by a one-warp planner.
constexpr int kSelfPlanMaxBatch = 32;
// One-warp planner: block-table entries each checking warp covers.
constexpr int kCheckEntriesPerWarp = 2048;

// The plan's arithmetic, shared by every place that computes it (the planner
// kernel's paths and the decode kernel's own plan), so that they agree exactly.
// Sequence of length L: valid when q_len <= L <= 64 * max_pages; n pages; cost
// n + kSeqOverhead units (0 when invalid or empty).
__host__ __device__ inline void plan_seq(int L, int q_len, int max_pages, bool& ok, int& n, int& cost) {
  ok = L >= q_len && L <= max_pages * kPage;
  n = ok ? (L + kPage - 1) / kPage : 0;
  cost = n > 0 ? n + kSeqOverhead : 0;
}
// Cost units per cluster for a line of `total` units over c_use clusters.
__host__ __device__ inline int plan_payload(int total, int c_use) {
  const int payload = (total + c_use - 1) / c_use;
  return payload < kMinPayload ? kMinPayload : payload;
}
__host__ __device__ inline int plan_clusters(int total, int payload) {
  return total > 0 ? (total + payload - 1) / payload : 0;
}
// First cluster and number of clusters holding the pages of a sequence whose
// cost interval starts at `start` and holds n > 0 pages.
__host__ __device__ inline void plan_split(int start, int n, int payload, int& first, int& splits) {
  const int ps = start + kSeqOverhead;
  first = ps / payload;
  splits = (ps + n - 1) / payload - first + 1;
}
#ifdef __CUDACC__
__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}
#endif

// Device error flag bits (workspace header word 0).
constexpr int kFlagTimeout = 1;      // a bounded wait ran out; the kernel gave up
constexpr int kFlagBadSeqlen = 2;    // L_b < q_len or L_b > max_pages * 64
constexpr int kFlagBadPage = 4;      // block-table entry outside [0, num_pages)
constexpr int kFlagBadPrefix = 8;    // cascade: a sequence's prefix pages are not the shared ones
constexpr int kFlagPlanMismatch = 16;  // a self-planned decode launch's plan differs from the planner's

// Workspace header words.
enum : int {
  kHdrFlag = 0,
  kHdrClusters = 1,   // active clusters per row tile
  kHdrPayload = 2,    // cost units per cluster
  kHdrTotal = 3,      // total cost units
  kHdrSlots = 4,      // partial slots used
  kHdrListed = 5,     // sequences the combine kernel visits (split or invalid)
  kHdrCombineCtas = 6,  // combine work items (virtual CTAs) over all listed sequences
  kHdrChecks = 7,     // planner CTAs that range-checked the block table (0: not checked)
  kHdrCheck0 = 8,     // [kMaxCheckCtas] per checking CTA: 1 if it found an entry out of range
  kHdrWords = 64,
};

// Per-sequence plan record (int32 x 8).
enum : int {
  kSeqStart = 0,    // exclusive prefix of cost units before this sequence
  kSeqPages = 1,    // pages of the sequence (0 when invalid)
  kSeqFirstC = 2,   // first cluster that holds one of its pages
  kSeqSplits = 3,   // number of clusters that hold its pages
  kSeqSlot = 4,     // first partial slot (valid when splits > 1)
  kSeqLen = 5,      // L_b as read
  kSeqWords = 8,
};

struct WsLayout {
  size_t first_b_off;   // int32 [c_max]: first sequence each cluster touches
  size_t seq_off;       // int32 [batch][8]
  size_t list_off;      // int32 [batch]: listed sequences (splits != 1), in batch order
  size_t vcp_off;       // int32 [batch]: inclusive prefix of combine work items per listed sequence
  size_t plse_off;      // float [max_slots][row_tiles][128]
  size_t po_off;        // float [max_slots][row_tiles][128][512]
  size_t total;
  int max_slots;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline WsLayout ws_layout(int batch, int row_tiles, int c_max) {
  WsLayout w;
  size_t off = kHdrWords * 4;
  w.first_b_off = off;
  off = align_up(off + 4 * static_cast<size_t>(c_max), 16);
  w.seq_off = off;
  off = align_up(off + 4 * static_cast<size_t>(kSeqWords) * batch, 16);
  w.list_off = off;
  off = align_up(off + 4 * static_cast<size_t>(batch), 16);
  w.vcp_off = off;
  off = align_up(off + 4 * static_cast<size_t>(batch), 256);
  w.max_slots = c_max + batch;
  w.plse_off = off;
  off = align_up(off + 4 * static_cast<size_t>(w.max_slots) * row_tiles * kRowsPerTile, 256);
  w.po_off = off;
  off += 4 * static_cast<size_t>(w.max_slots) * row_tiles * kRowsPerTile * kDv;
  w.total = align_up(off, 256);
  return w;
}

// Split combine work decomposition. One task = one query row x one 128-column
// chunk of a listed sequence; a sequence cut into s pieces gives each task
// combine_warps(s) warps (each summing a share of the pieces), and 8 warps
// make one work item (a CTA's worth), so each warp keeps at most ~9 partial
// rows in flight.
constexpr int kCombineWarps = 8;
constexpr int kCombineMaxSplits = 256;   // pieces per sequence the combine supports
__host__ __device__ inline int combine_warps(int splits) {
  return splits <= 8 ? 1 : splits <= 16 ? 2 : splits <= 32 ? 4 : 8;
}
__host__ __device__ inline int combine_items(int splits, int rows) {
  return (rows * 4 * combine_warps(splits) + kCombineWarps - 1) / kCombineWarps;
}

struct PlanParams {
  const int32_t* seqlens;
  const int32_t* block_table;   // [batch, max_pages] or nullptr (no page-id check)
  long long num_pages;          // pool size the block table must index into
  int check_ctas;               // CTAs 1..check_ctas of the grid range-check the block table
  int32_t* ws;
  int batch, max_pages, q_len, row_tiles;
  int rows;    // query rows per sequence (q_len * heads)
  int c_max;   // clusters per row tile the workspace layout and grid are sized for
  int c_use;   // clusters per row tile to spread work over (<= c_max)
  int warp_plan;   // 1: one-warp planner (batch <= kSelfPlanMaxBatch), checking warps of kCheckEntriesPerWarp
  long long* trace;   // phase timestamps (instrumented builds only; else unused)
};

struct DecodeParams {
  const void* q;                // bf16 [batch * q_len * heads, 576]
  const void* kv_cache;         // page pool (fp8: for the per-token scales)
  const int32_t* block_table;   // [batch, max_pages]
  const int32_t* seqlens;       // [batch]
  uint16_t* out;                // bf16 [batch * q_len * heads, 512]
  float* lse;                   // [batch * q_len * heads]
  int32_t* ws;                  // workspace base
  int batch, max_pages, q_len, heads, rows, row_tiles, c_max;
  int tile_rows;                // query rows per tile: 64 or 128
  int fp8;                      // cache is fp8-e4m3 pages with per-token fp32 scales
  long long num_pages;
  float scale_log2;             // softmax scale * log2(e)
  int self_plan;                // 1: each CTA derives the plan from seqlens (batch <= kSelfPlanMaxBatch)
  int c_use;                    // the planner's cluster budget (used when self_plan)
  unsigned long long timeout_ns;
  long long* trace;             // phase timestamps (instrumented builds only; else unused)
};

struct CombineParams {
  const int32_t* ws;
  uint16_t* out;
  float* lse;
  int batch, rows, row_tiles, c_max;
  int tile_rows;                // query rows per tile: 64 or 128
  int grid;                     // CTAs to launch (a fixed multiple of the SM count)
  long long* trace;             // phase timestamps (instrumented builds only; else unused)
};

struct AppendParams {
  const uint16_t* src;          // bf16 [batch * q_len, 576]: the new tokens' latent rows
  void* cache;                  // page pool (bf16 pages, or fp8 codes + token scales)
  const int32_t* block_table;   // [batch, max_pages]
  const int32_t* seqlens;       // [batch], counting the new tokens
  int32_t* flag;                // device word for kFlagBadSeqlen / kFlagBadPage, or nullptr
  long long num_pages;
  int batch, max_pages, q_len;
  int fp8;
};

struct ProjParams {
  const uint16_t* in;           // absorb: q [n_tokens, heads, 192] (for the RoPE pass-through); project: unused
  uint16_t* out;                // absorb: q~ [n_tokens, heads, 576]; project: y [n_tokens, heads, 128]
  int32_t* flag;                // device word for kFlagTimeout, or nullptr
  int n_tokens, heads;
  int out_row;                  // elements per output row (576 or 128)
  unsigned long long timeout_ns;
};

struct CascadeParams {
  const int32_t* seqlens;       // [batch]
  const int32_t* block_table;   // [batch, max_pages]
  int32_t* seqlens_suffix;      // [batch] written: L_b - P (0 when invalid)
  int32_t* seqlen_prefix;       // [1] written: P
  int32_t* flag;                // cascade flag word (kFlagBadSeqlen / kFlagBadPrefix)
  int batch, max_pages, q_len, prefix_len;
};

struct MergeParams {
  const uint16_t* out_a;        // bf16 [rows, 512] (prefix pass)
  const float* lse_a;
  const uint16_t* out_b;        // bf16 [rows, 512] (suffix pass)
  const float* lse_b;
  uint16_t* out;                // bf16 [rows, 512]
  float* lse;
  long long rows;
  int32_t* flag_prefix;         // flag words: folded into flag_prefix
  const int32_t* flag_suffix;
  const int32_t* flag_prep;
};

// Instrumented builds (-DMLA_TRACE) stamp %globaltimer at kernel boundaries into
// trace[kTraceStepBase + k]: 0/1 planner entry/exit, 2 first combine CTA entry,
// 3 last combine CTA exit, 4 first combine CTA past its grid-dependency wait,
// 5 last block-table checking CTA of the planner done.
constexpr int kTraceStepBase = 8192 + 16 * 1024;

}  // namespace mla
