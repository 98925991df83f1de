// K1: MLA decode main kernel over a paged latent cache (sm_100a).
//
// Work unit: one cluster of two CTAs owns a contiguous range of (sequence,
// page) work from the planner (K0) for one tile of kRows query rows (t, h).
// The pair splits the work so that neither CTA duplicates tensor-core flops
// and both fit their state in tensor memory (512 columns per SM):
//
//   * PV is split along V's 512 columns: CTA r accumulates O[:, 256r:256r+256]
//     (TMEM columns 0..255).
//   * QK^T is split along the 576-wide contraction: CTA r contracts latent
//     columns [256r, 256r+256) - the same columns it needs as its V half - plus
//     rope columns [512+32r, 512+32r+32). Its latent query slice lives in TMEM
//     (columns 384..511, the MMA's A operand); the rope slice stays in shared
//     memory. The two partial score tiles are summed through distributed shared
//     memory: staged in the sender's shared memory, then one bulk
//     shared::cluster copy per 4 KB slice, counted on the receiver's mbarrier.
//
// Softmax, bf16 cache (the pair path): the CTAs take alternate tiles. CTA r
// owns the tiles g with g % 2 == r: its exchange warps send the other tiles'
// partial S to the peer, and its softmax warps sum the peer's partial into
// their own for the tiles they own, apply the online softmax, and copy the P
// rows back to the peer. The running max of the previous tile reaches the
// owner through the peer early in the peer's softmax. Each CTA keeps the row
// sums of its own tiles; the pair adds them at the segment's epilogue.
// Softmax, fp8 cache: both CTAs compute every tile's softmax on the summed
// scores (bit-identical decisions), at 64 rows with the two warps of a lane
// quarter taking alternate tiles, at 128 rows splitting each tile's tokens.
//
// Per 64-token page (one KV tile) and CTA:
//   TMA warp  : block_table[b, i] -> this CTA's columns of the page. bf16 cache:
//               4 latent boxes of 64x64 (128B swizzle) and this CTA's 32 rope
//               columns (64B swizzle), straight into a bf16 stage. fp8 cache:
//               the e4m3 codes (2 latent boxes of 64x128, rope box 64x64) and
//               the 64 fp32 token scales into a raw stage, which converter
//               warps expand exactly into a bf16 stage.
//   QK thread : S_r = Q_r K_r^T, 16 tcgen05.mma (A from TMEM) + 2 rope ones
//               (A from shared memory), M128 N64 K16, into a double S buffer.
//   PV thread : O_r += P V_r, 4 tcgen05.mma M128 N256 K16, V read MN-major from
//               the page tile. QK and PV have their own issuing threads.
//   softmax warps (two per row quarter, one query row per thread): query
//               rows into TMEM at each segment start, fp8 token scales on S,
//               causal mask among the q_len draft tokens, online softmax in the
//               log2 domain (lazy rescale), P (bf16; fp8: times the token
//               scale) to shared memory, rare O rescales in TMEM, epilogue O/l
//               (bf16 out, or fp32 partial for split sequences) and lse.
//
// Instantiations: kRows = 64 for steps with at most 64 query rows (the MMA still
// runs M = 128; rows 64..127 are never read) and kRows = 128; bf16 or fp8 cache.
//
// The pages name the kernel (evermx.com, "TokenSpeed: speed-of-light LLM
// inference engine for agentic workloads", section "Pluggable Kernel
// Registry") but give no design; this one is written for B200 from scratch.
#include <cmath>

#include <cuda_bf16.h>

#include "mla_common.cuh"
#include "mla_launch.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr int kBoxes = 5;                          // 4 latent boxes + 1 rope box (bf16 stage)
constexpr int kKvBoxBytes = kPage * 128;           // 64 tokens x 64 bf16
// fp8: token scales (256 B) follow the boxes of a bf16 stage, 1 KB aligned.
constexpr int kScaleOff = kBoxes * kKvBoxBytes;
// A stage holds the 4 latent boxes of this CTA's 256 columns and the rope box:
// all 64 rope columns (128-byte swizzle), or with a narrow rope only this
// CTA's 32 (64-byte swizzle).
template <bool kFp8, bool kNarrow>
constexpr int stage_bytes() { return 4 * kKvBoxBytes + (kNarrow ? kKvBoxBytes / 2 : kKvBoxBytes) + (kFp8 ? 1024 : 0); }

// Raw fp8 stage: 2 latent boxes [64 tok x 128 codes] (128B swizzle), rope box
// [64 tok x 64 codes] (no swizzle), 64 fp32 token scales.
constexpr int kRawLatBytes = kPage * 128;          // 8 KB
constexpr int kRawRopeOff = 2 * kRawLatBytes;
constexpr int kRawScaleOff = kRawRopeOff + kPage * 64;
constexpr int kRawStageBytes = 21504;              // 16 KB + 4 KB + 256 B, 1 KB aligned
constexpr int kRawTx = 2 * kRawLatBytes + kPage * 64 + kPage * 4;

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;      // O half: columns [0, 256)
constexpr uint32_t kTmemS = 256;    // S double buffer: [256, 320), [320, 384)
constexpr uint32_t kTmemQ = 384;    // this CTA's 256 latent query columns, packed bf16x2: [384, 512)

constexpr unsigned long long kDrainTimeoutNs = 200ull * 1000 * 1000;

// Phase tracing for performance analysis: compiled in only with -DMLA_TRACE.
// Records clock64() of cluster 0, CTA rank 0, into p.trace (8192 entries):
//   [0, 2048)    softmax warp 0 lane 0: 16 stamps per tile (first 128 tiles)
//   [2048, 4096) softmax warp 1 lane 0: same
//   [4096, 6144) QK / PV threads: 4 stamps per tile (QK start/end, PV start/end)
//   [6144, 8192) TMA thread: 1 stamp per tile (load issue)
#ifdef MLA_TRACE
#define MLA_TRACE_AT(cond, idx)                                                          \
  do {                                                                                   \
    if ((cond) && blockIdx.x == 0 && p.trace != nullptr && (idx) >= 0 && (idx) < 8192)  \
      p.trace[idx] = clock64();                                                          \
  } while (0)
// Timeline: %globaltimer (ns) of 16 events per CTA at [8192 + 16 * blockIdx.x, +16).
#define MLA_TL(cond, k)                                                                  \
  do {                                                                                   \
    if ((cond) && p.trace != nullptr && blockIdx.x < 1024)                               \
      p.trace[8192 + 16 * blockIdx.x + (k)] = static_cast<long long>(globaltimer_ns());  \
  } while (0)
#else
#define MLA_TRACE_AT(cond, idx) \
  do {                          \
  } while (0)
#define MLA_TL(cond, k) \
  do {                  \
  } while (0)
#endif

constexpr int align1k(int x) { return (x + 1023) / 1024 * 1024; }

template <int kRows, bool kFp8>
struct Cfg {
  // Softmax warps: two per TMEM lane quarter. Warp w may only touch TMEM lanes
  // 32*(w%4)..+31, so the softmax warps are {0..7} (128 rows) or {0,1,4,5}
  // (64 rows); the other roles take the rest.
  static constexpr int kQuarters = kRows / 32;
  static constexpr int kSoftmaxThreads = 2 * kRows;
  // bf16 cache: the pair's CTAs take alternate tiles' softmax (CTA r the tiles
  // g with g % 2 == r; the two warps of a quarter split the tile's tokens); the
  // other CTA's exchange warps send it their partial S and receive P back, so
  // no tile's softmax is computed twice.
  // fp8 cache: both CTAs compute every tile's softmax; at 64 rows the two warps
  // of a lane quarter take alternate tiles (ping-pong), at 128 they split each
  // tile's tokens. (The pair protocol also runs fp8 correctly, but at 128 rows
  // it leaves room for a single converter warp within 16 warps / 128 registers,
  // and conversion then bounds the tile rate: 2x slower.)
  static constexpr bool kPair = !kFp8;
  static constexpr bool kPingPong = !kPair && kRows == 64;
  static constexpr int kTileThreads = kPingPong ? kRows : 2 * kRows;   // threads that process one tile
  static constexpr int kPBufs = (kPingPong || kPair) ? 2 : 1;   // P-ready barriers (by tile parity)
  static constexpr int kPSmem = kPingPong ? 2 : 1;              // P tiles in shared memory
  // Pair path: one exchange warp per lane quarter moves the partial S of the
  // peer's tiles, so the softmax warps only receive.
  static constexpr bool kXchg = kPair;
  static constexpr int kXchgWarp0 = 8;
  static constexpr int kXchgWarps = kXchg ? kQuarters : 0;
  static constexpr int kTmaWarp = kRows == 128 ? 8 + kXchgWarps : 2;
  static constexpr int kQkWarp = kRows == 128 ? kTmaWarp + 1 : 3;
  static constexpr int kPvWarp = kRows == 128 ? kTmaWarp + 2 : 6;
  // 64 rows: warp 7 is idle (and the converters start after the exchange warps)
  static constexpr int kCvtWarp0 = kRows == 128 ? kTmaWarp + 3 : (kXchg ? kXchgWarp0 + kXchgWarps : 7);
  // fp8 converters (a pair-path fp8 build at 128 rows would have room for one)
  static constexpr int kCvtWarps = kFp8 ? ((kPair && kRows == 128) ? 1 : 4) : 0;
  static constexpr int kCvtThreads = kCvtWarps * 32;
  // Chunks of 16 codes (of 10 per converter thread and tile) expanded into
  // registers before the bf16 stage is free: more overlaps more of the wait, but
  // competes with the softmax warps for issue slots (measured best: 6 at 128
  // rows, 3 at 64; 7 at 128 rows was 4% slower than 6).
  static constexpr int kCvtAhead = kRows == 128 ? 6 : 3;
  // Pair path: QK(g) is issued after PV(g - kQkGate) (A/B, bf16: spec 128K and the
  // agentic batch -2.5%, the 50K step -1%; 2 was 30% slower, 4 in between; on the
  // fp8 split path the same gate cost 3%).
  static constexpr int kQkGate = kPair ? 3 : 0;
  // Pair path: P tiles in the 64-byte-swizzle K-major layout (tokens 0-31 of all
  // rows, then tokens 32-63), so that each softmax warp's part of a tile (32 rows
  // x 32 tokens) is one contiguous 2 KB block it can copy to the peer on its own.
  static constexpr bool kPSw64 = kPair;
  static_assert(kQkGate <= 4, "pvissued has 4 slots");
  static constexpr int kWarps = (kCvtWarp0 + kCvtWarps) > (kXchgWarp0 + kXchgWarps) ? (kCvtWarp0 + kCvtWarps)
                                                                                      : (kXchgWarp0 + kXchgWarps);
  static constexpr int kThreads = kWarps * 32;
  // Pair path: only this CTA's 32 rope columns of K and Q are loaded (64-byte
  // swizzle), and the exchange staging is one 4 KB slice per quarter, which
  // makes room for more KV stages (4 at 128 rows, 5 at 64). The stage ring
  // bounds the pair path's tile period (a stage lives from its TMA load to the
  // PV that reads it, across both CTAs' parts of the tile), so stages take
  // precedence over a second P tile.
  static constexpr bool kNarrowRope = kPair && !kFp8;
  static constexpr int kStageBytes = stage_bytes<kFp8, kNarrowRope>();
  // bf16 stages the MMAs read; raw fp8 stages the TMA fills (fp8 only).
  static constexpr int kStages = kFp8 ? 2 : (kPair ? (kRows == 64 ? 5 : 4) : 3);
  static constexpr int kRawStages = kFp8 ? 2 : 0;
  // Partial-S exchange buffers: two let tile g+1's exchange overlap tile g
  // (64-row ping-pong); the pair path needs one (each CTA receives every other tile).
  static constexpr int kXBufs = kPingPong ? 2 : 1;
  static constexpr int kQRopeBytes = kRows * (kNarrowRope ? 64 : 128);   // rope query box [kRows x 64 (32)] bf16
  // The PV MMA reads 128 rows of P (and the rope QK MMA 128 rows of the rope
  // query box); with 64 live rows the upper half of those reads lands in the
  // next buffer, which is harmless.
  static constexpr int kPBytes = kRows * kPage * 2;            // one P tile
  // One exchange buffer (and the staging buffer): [token half][kRows][32] fp32,
  // so that each warp's 32 rows x 32 tokens are one contiguous 4 KB slice.
  static constexpr int kXBytes = kRows * kPage * 4;
  static constexpr int kOffQR = 0;
  static constexpr int kOffKV = align1k(kOffQR + kQRopeBytes);
  static constexpr int kOffRaw = kOffKV + kStages * kStageBytes;
  static constexpr int kOffP = align1k(kOffRaw + kRawStages * kRawStageBytes);
  static constexpr int kOffX = align1k(kOffP + kPSmem * kPBytes);
  static constexpr int kOffXS = kOffX + kXBufs * kXBytes;
  static constexpr int kXSBufs = kPingPong ? 2 : 1;             // staging buffers
  // pair path: one 4 KB slice per quarter (the two token halves go one after the other)
  static constexpr int kXSBytes = kPair ? kRows * 32 * 4 : kXSBufs * kXBytes;
  static constexpr int kOffRed = kOffXS + kXSBytes;          // pair reductions: [2 tiles][2 halves][kRows] + [2][kRows]
  // pair path adds: m of the latest tiles [2][kRows], m from the peer [2][kRows],
  // m staging [kRows], row sums from the peer [kRows], row-sum staging [kRows]
  static constexpr int kRedBytes = align1k((kPair ? 13 : 6) * kRows * 4);
  // the sequence records of a self-planned launch: [kSelfPlanMaxBatch][kSeqWords]
  static constexpr int kOffPlan = kOffRed + kRedBytes;
  static constexpr int kPlanBytes = kSelfPlanMaxBatch * kSeqWords * 4;
  static constexpr int kOffBar = kOffPlan + kPlanBytes;
  static constexpr int kSmemBytes = kOffBar + 1024 + 1024;  // barriers + alignment slack
  static_assert(kSmemBytes <= 232448, "shared memory");
  static __device__ __forceinline__ bool is_softmax(int w) { return w < 8 && (w & 3) < kQuarters; }
  static __device__ __forceinline__ bool is_xchg(int w) { return w >= kXchgWarp0 && w < kXchgWarp0 + kXchgWarps; }
};

template <int kStages, int kRawStages>
struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t rawfull[kRawStages > 0 ? kRawStages : 1];
  uint64_t rawempty[kRawStages > 0 ? kRawStages : 1];
  uint64_t qfull, qtm, qempty;
  uint64_t qissued;                            // pair path: the first segment's query loads are issued
  uint64_t sfull[2], sfree[2];
  uint64_t pfull[2], pvdone[2];               // [P buffer] (one buffer unless ping-pong)
  uint64_t mready[4];                          // ping-pong: running max handed between a quarter's warps
  uint64_t xfull[2][4][2], xempty[2][4][2];   // [exchange buffer][lane quarter][token half]
  uint64_t mhfull[2][4];                       // pair path: running max from the peer, [slot][quarter]
  uint64_t epi[4];                             // pair path: the peer's epilogue is done with its P rows
  uint64_t lfull[4];                           // pair path: row sums from the peer
  uint64_t pairb[4];                           // pair path: the two softmax warps of a quarter meet (bounded)
  uint64_t drain_qk, drain_pv;
  uint64_t pvissued[4];                        // [tile % 4]: the PV of the tile has been issued
  uint32_t tmem_base;
  int abort;
  int flags;                                   // device-flag bits raised by this CTA (written out at the end)
  int plan_hdr[4];                             // self-planned launch: clusters, payload, total, first sequence
};

// Walks the (sequence, page range) segments of cluster position range [x0, x1).
struct SegIter {
  const int32_t* seq;
  int batch, x0, x1, b;
  __device__ bool next(int& ob, int& lo, int& hi) {
    while (b < batch) {
      const int32_t* s = seq + static_cast<size_t>(b) * kSeqWords;
      const int ps = s[kSeqStart] + kSeqOverhead;
      const int n = s[kSeqPages];
      if (ps >= x1) {
        b = batch;
        return false;
      }
      const int l = max(x0, ps) - ps;
      const int h = min(x1, ps + n) - ps;
      const int cur = b++;
      if (h > l) {
        ob = cur;
        lo = l;
        hi = h;
        return true;
      }
    }
    return false;
  }
};

// Walks the tiles (pages) of a cluster's segments in order.
struct TileIter {
  SegIter it;
  int b = 0, lo = 0, hi = 0, i = 0, seg = -1;
  bool valid = false;
  __device__ void start() {
    valid = it.next(b, lo, hi);
    i = lo;
    seg = valid ? 0 : -1;
  }
  __device__ void advance() {
    if (++i < hi) return;
    valid = it.next(b, lo, hi);
    i = lo;
    if (valid) ++seg;
  }
  __device__ bool first() const { return i == lo; }
  __device__ bool last() const { return i == hi - 1; }
};

// The step's plan as the planner kernel computes it (same arithmetic), by one
// warp from the sequence lengths of a batch of at most kSelfPlanMaxBatch (lane
// b = sequence b): the per-sequence records the iterators and the epilogue read
// go to `seqs` ([batch][kSeqWords], shared memory), and the clusters in use, the
// payload, the total cost and this cluster's first sequence to `hdr4`.
__device__ void self_plan_warp(const DecodeParams& p, int c_idx, int32_t* seqs, int* hdr4, int lane) {
  const bool in = lane < p.batch;
  int L = 0, n = 0, cost = 0;
  if (in) {
    L = p.seqlens[lane];
    bool ok;
    plan_seq(L, p.q_len, p.max_pages, ok, n, cost);
  }
  const int incl = warp_inclusive_scan(cost, lane);
  const int start = incl - cost;
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  const int payload = plan_payload(total, p.c_use);
  const int clusters = plan_clusters(total, payload);
  int splits = 0, first = 0;
  if (n > 0) plan_split(start, n, payload, first, splits);
  const int sv = splits > 1 ? splits : 0;
  const int slot = warp_inclusive_scan(sv, lane) - sv;
  if (in) {
    int32_t* s = seqs + lane * kSeqWords;
    s[kSeqStart] = start;
    s[kSeqPages] = n;
    s[kSeqLen] = L;
    s[kSeqFirstC] = first;
    s[kSeqSplits] = splits;
    s[kSeqSlot] = slot;
  }
  const int x0 = c_idx < clusters ? c_idx * payload : 0;
  const unsigned m = __ballot_sync(0xffffffffu, in && start + cost > x0);
  if (lane == 0) {
    hdr4[0] = clusters;
    hdr4[1] = payload;
    hdr4[2] = total;
    hdr4[3] = (c_idx < clusters && m != 0u) ? __ffs(m) - 1 : p.batch;
  }
}

__device__ __forceinline__ int box_col(int rank, int box) { return box < 4 ? rank * 256 + box * 64 : 512; }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Byte offset of the 16-byte chunk `chunk` of row `row` in a 128B-swizzled tile
// whose rows are 128 bytes (8-row, 1024-byte atoms).
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
}

// Epilogue stores. A warp holds 32 rows (one per lane) of kRowBytes (64 or
// 128) bytes each in registers; stored directly, every store instruction would
// touch 32 rows. Instead the rows pass through a shared-memory tile (16-byte
// chunks XOR-swizzled by row, conflict-free both ways) and come back out so
// that each store instruction writes whole 64- or 128-byte row segments.
// Rows >= valid_rows are not written.
template <int kRowBytes>
__device__ __forceinline__ void store_rows(uint32_t stg, int lane, const uint32_t (&w)[kRowBytes / 4], char* dst0,
                                           size_t stride, int valid_rows) {
  constexpr int kChunks = kRowBytes / 16;
  auto swz = [](int r) { return kChunks == 8 ? (r & 7) : ((r >> 1) & 3); };
#pragma unroll
  for (int v = 0; v < kChunks; ++v)
    st_shared_v4_u32(stg + lane * kRowBytes + ((v ^ swz(lane)) << 4), w[4 * v], w[4 * v + 1], w[4 * v + 2],
                     w[4 * v + 3]);
  __syncwarp();
  const int c16 = lane % kChunks;
#pragma unroll
  for (int k = 0; k < kChunks; ++k) {
    const int r = k * (32 / kChunks) + lane / kChunks;
    const float4 v = ld_shared_v4(stg + r * kRowBytes + ((c16 ^ swz(r)) << 4));
    if (r < valid_rows) *reinterpret_cast<float4*>(dst0 + r * stride + c16 * 16) = v;
  }
  __syncwarp();
}

// Writes a warp's 32 rows x 128 columns of O (TMEM columns tcol.., lane = row)
// times inv: bf16 into `out` rows (stride kDv), or fp32 into partial rows.
// The staging tile is 32 x kRowBytes bytes.
template <bool kBf16, int kRowBytes>
__device__ __forceinline__ void store_o_rows(uint32_t tcol, uint32_t stg, int lane, float inv, char* dst0,
                                             int valid_rows) {
  constexpr int kWords = kRowBytes / 4;            // 32-bit words per staged row
  constexpr int kWordsPerLoad = kBf16 ? 16 : 32;   // words from one 32-column TMEM load
  uint32_t w[kWords];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    float a[32];
    tmem_ld32(tcol + 32u * g, a);
    tc_wait_ld();
#pragma unroll
    for (int k = 0; k < kWordsPerLoad; ++k) {
      const int n = g * kWordsPerLoad + k;         // word index along the 128 columns
      w[n % kWords] = kBf16 ? pack_bf16x2(a[2 * k] * inv, a[2 * k + 1] * inv) : __float_as_uint(a[k] * inv);
      if ((n + 1) % kWords == 0)
        store_rows<kRowBytes>(stg, lane, w, dst0 + (n / kWords) * kRowBytes, kDv * (kBf16 ? 2 : 4), valid_rows);
    }
  }
}

template <int kRows, bool kFp8>
__global__ void __launch_bounds__(Cfg<kRows, kFp8>::kThreads, 1)
    mla_decode_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                      const __grid_constant__ CUtensorMap tm_kv2, const DecodeParams p) {
  using C = Cfg<kRows, kFp8>;
  constexpr int kStages = C::kStages;
  constexpr int kStageBytes = C::kStageBytes;
  constexpr int kRaw = C::kRawStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars<kStages, kRaw>* bars = reinterpret_cast<Bars<kStages, kRaw>*>(smem + C::kOffBar);
  static_assert(sizeof(Bars<kStages, kRaw>) <= 1024, "the barrier block has 1 KB");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cluster = blockIdx.x >> 1;
  const int r_tile = cluster / p.c_max;
  const int c_idx = cluster % p.c_max;
  MLA_TL(threadIdx.x == 0, 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], kFp8 ? C::kCvtThreads : 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int s = 0; s < kRaw; ++s) {
      mbar_init(&bars->rawfull[s], 1);
      mbar_init(&bars->rawempty[s], C::kCvtThreads);
    }
    mbar_init(&bars->qfull, 1);
    mbar_init(&bars->qtm, C::kTileThreads);
    mbar_init(&bars->qissued, C::kTileThreads);
    mbar_init(&bars->qempty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->sfull[i], 1);
      if constexpr (C::kPair) {
        // S buffer / P parity `rank`: this CTA's softmax threads; the other: its exchange warps
        const bool own = static_cast<uint32_t>(i) == rank;
        mbar_init(&bars->sfree[i], own ? C::kTileThreads : kRows);
        mbar_init(&bars->pfull[i], own ? C::kTileThreads : kRows);
        mbar_init(&bars->pvdone[i], 2);   // tiles of parity i: the PVs of both CTAs
      } else {
        mbar_init(&bars->sfree[i], C::kTileThreads);
        mbar_init(&bars->pfull[i], C::kTileThreads);
        mbar_init(&bars->pvdone[i], 1);
      }
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bars->mhfull[0][i], 1);
      mbar_init(&bars->mhfull[1][i], 1);
      mbar_init(&bars->epi[i], 1);
      mbar_init(&bars->lfull[i], 1);
      mbar_init(&bars->pairb[i], 64);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&bars->mready[i], 32);
    for (int x = 0; x < 2; ++x) {
      for (int i = 0; i < 4; ++i) {
        for (int h = 0; h < 2; ++h) {
          mbar_init(&bars->xfull[x][i][h], 1);
          mbar_init(&bars->xempty[x][i][h], 1);
        }
      }
    }
    mbar_init(&bars->drain_qk, 1);
    mbar_init(&bars->drain_pv, 1);
    for (int i = 0; i < 4; ++i) mbar_init(&bars->pvissued[i], 1);
    bars->abort = 0;
    bars->flags = 0;
    fence_mbar_init_cluster();
  }
  if (warp == C::kTmaWarp && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_kv);
    if (kFp8 || C::kNarrowRope) prefetch_tensormap(&tm_kv2);
  }
  if (warp == C::kQkWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (p.self_plan && warp == C::kPvWarp)
    self_plan_warp(p, c_idx, reinterpret_cast<int32_t*>(smem + C::kOffPlan), bars->plan_hdr, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // the peer's barriers are initialised before any remote arrive
  MLA_TL(threadIdx.x == 0, 1);

  const WsLayout w = ws_layout(p.batch, p.row_tiles, p.c_max);
  int32_t* hdr = p.ws;
  const int32_t* seq;
  int clusters, payload = 0, total = 0, fb = p.batch;
  if (p.self_plan) {
    // The plan derived above: this launch need not wait for the planner kernel
    // (it waits before its first global store and before writing the flag).
    seq = reinterpret_cast<const int32_t*>(smem + C::kOffPlan);
    clusters = bars->plan_hdr[0];
    if (c_idx < clusters) {
      payload = bars->plan_hdr[1];
      total = bars->plan_hdr[2];
      fb = bars->plan_hdr[3];
    }
  } else {
    // The set-up above overlaps the planner; the plan is read only after it completes.
    pdl_wait();
    seq = reinterpret_cast<const int32_t*>(reinterpret_cast<const char*>(p.ws) + w.seq_off);
    const int32_t* first_b = reinterpret_cast<const int32_t*>(reinterpret_cast<const char*>(p.ws) + w.first_b_off);
    clusters = hdr[kHdrClusters];
    if (c_idx < clusters) {
      payload = hdr[kHdrPayload];
      total = hdr[kHdrTotal];
      fb = first_b[c_idx];
    }
  }
  pdl_launch_dependents();
  MLA_TL(threadIdx.x == 0, 2);
  // Both CTAs of a cluster see the same plan, so both go idle together.
  const bool active = c_idx < clusters && r_tile < p.row_tiles;
  const int x0 = active ? c_idx * payload : 0;
  const int x1 = active ? min(x0 + payload, total) : 0;
  const int b_first = active ? fb : p.batch;   // an idle cluster walks no segment
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  const unsigned long long tmo = p.timeout_ns;

  // Outstanding-work trackers for the abort drain.
  int tma_last_g = -1, tma_q_issued = 0;
  bool mma_issued_any = false, pv_issued_any = false;

  if (warp == C::kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      SegIter it{seq, p.batch, x0, x1, b_first};
      int g = 0, segi = 0, b, lo, hi;
      bool ok = true;
      while (ok && it.next(b, lo, hi)) {
        // rope query box of this segment (the latent slice goes to TMEM via the softmax warps)
        if (segi > 0 && !mbar_wait(&bars->qempty, (segi - 1) & 1, tmo, abort_flag)) break;
        mbar_arrive_expect_tx(&bars->qfull, C::kQRopeBytes);
        tma_load_2d(smem + C::kOffQR, &tm_q, &bars->qfull, C::kNarrowRope ? 512 + 32 * static_cast<int>(rank) : 512,
                    b * p.rows + r_tile * kRows);
        tma_q_issued = segi + 1;
        const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages;
        int phys_next = bt[lo];
        if (C::kPair && segi == 0 && !mbar_wait(&bars->qissued, 0, tmo, abort_flag)) break;
        for (int i = lo; i < hi; ++i, ++g) {
          int phys = phys_next;
          if (i + 1 < hi) phys_next = bt[i + 1];   // prefetch the next page id
          if (phys < 0 || phys >= p.num_pages) {
            atomicOr(&bars->flags, kFlagBadPage);
            phys = 0;
          }
          MLA_TRACE_AT(g < 2048, 6144 + g);
          MLA_TL(g == 0, 3);
          MLA_TL(true, 15);
          if constexpr (!kFp8) {
            const int s = g % kStages;
            if (g >= kStages && !mbar_wait(&bars->empty[s], ((g / kStages) - 1) & 1, tmo, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
            uint8_t* dst = smem + C::kOffKV + s * kStageBytes;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tma_load_3d(dst + k * kKvBoxBytes, &tm_kv, &bars->full[s], box_col(rank, k), 0, phys);
            if constexpr (C::kNarrowRope)
              tma_load_3d(dst + 4 * kKvBoxBytes, &tm_kv2, &bars->full[s], 512 + 32 * static_cast<int>(rank), 0, phys);
            else
              tma_load_3d(dst + 4 * kKvBoxBytes, &tm_kv, &bars->full[s], box_col(rank, 4), 0, phys);
          } else {
            const int r = g % kRaw;
            if (g >= kRaw && !mbar_wait(&bars->rawempty[r], ((g / kRaw) - 1) & 1, tmo, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bars->rawfull[r], kRawTx);
            uint8_t* dst = smem + C::kOffRaw + r * kRawStageBytes;
            tma_load_3d(dst, &tm_kv, &bars->rawfull[r], rank * 256, 0, phys);
            tma_load_3d(dst + kRawLatBytes, &tm_kv, &bars->rawfull[r], rank * 256 + 128, 0, phys);
            tma_load_3d(dst + kRawRopeOff, &tm_kv2, &bars->rawfull[r], 512, 0, phys);
            const uint8_t* page = reinterpret_cast<const uint8_t*>(p.kv_cache) +
                                  static_cast<size_t>(phys) * kFp8PageBytes + kPage * kDqk;
            bulk_load_g2s(dst + kRawScaleOff, page, kPage * 4, &bars->rawfull[r]);
          }
          tma_last_g = g;
        }
        ++segi;
      }
    }
  } else if (warp == C::kQkWarp) {
    // ------------------------------------------------------------ QK issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, false, false);
      // Base descriptors; every K-step / box offset is added to the start-address
      // field (16-byte units, no carry out of its 14 bits below 256 KB).
      const uint64_t dQR = smem_desc_sw128(smem_u32(smem + C::kOffQR), 16, 1024);
      const uint64_t dKV = smem_desc_sw128(smem_u32(smem + C::kOffKV), 16, 1024);
      const uint64_t dQR64 = smem_desc_sw64(smem_u32(smem + C::kOffQR), 16, 512);
      const uint64_t dKV64 = smem_desc_sw64(smem_u32(smem + C::kOffKV), 16, 512);
      TileIter qk{SegIter{seq, p.batch, x0, x1, b_first}};
      qk.start();
      int seg_ready = -1;
      for (int g = 0; qk.valid; qk.advance(), ++g) {
        const int s = g % kStages;
        if (seg_ready < qk.seg) {
          if (!mbar_wait(&bars->qfull, qk.seg & 1, tmo, abort_flag)) break;
          if (!mbar_wait(&bars->qtm, qk.seg & 1, tmo, abort_flag)) break;
          seg_ready = qk.seg;
        }
        if (!mbar_wait(&bars->full[s], (g / kStages) & 1, tmo, abort_flag)) break;
        if (g >= 2 && !mbar_wait(&bars->sfree[g & 1], ((g >> 1) - 1) & 1, tmo, abort_flag)) break;
        // Pair path: QK(g) waits until PV(g - 3) has been issued, so that the tensor
        // pipe takes that PV (on the pair's P-handoff chain) before this tile's 18
        // QK MMAs rather than behind them. (pvissued has 4 slots: a waiter on tile
        // g - 3 can never see the slot's next phase, PV(g + 1), which needs QK(g + 1).)
        if constexpr (C::kQkGate > 0) {
          if (g >= C::kQkGate &&
              !mbar_wait(&bars->pvissued[(g - C::kQkGate) & 3], ((g - C::kQkGate) >> 2) & 1, tmo, abort_flag))
            break;
        }
        tc_fence_after();
        MLA_TRACE_AT(g < 512, 4096 + 4 * g);
        MLA_TL(g == 0, 4);
        MLA_TL(true, 13);
        const uint32_t dS = tmem + kTmemS + 64u * (g & 1);
        const uint64_t dK = dKV + static_cast<uint64_t>((s * kStageBytes) >> 4);
#pragma unroll
        for (int k = 0; k < 16; ++k)   // latent: A = query slice in TMEM (8 columns per K-step)
          umma_bf16_ts(dS, tmem + kTmemQ + 8u * k,
                       dK + static_cast<uint64_t>(((k >> 2) * kKvBoxBytes + (k & 3) * 32) >> 4), idesc_qk,
                       k != 0 ? 1u : 0u);
        if constexpr (C::kNarrowRope) {   // the rope boxes hold only this CTA's 32 columns (64-byte swizzle)
          const uint64_t dK64 = dKV64 + static_cast<uint64_t>((s * kStageBytes + 4 * kKvBoxBytes) >> 4);
          umma_bf16_ss(dS, dQR64, dK64, idesc_qk, 1u);
          umma_bf16_ss(dS, dQR64 + 2, dK64 + 2, idesc_qk, 1u);
        } else {   // this CTA's 32 rope columns: K-steps 2r, 2r+1 of the rope boxes
          const uint32_t rq = (64 * rank) >> 4, rk = (4 * kKvBoxBytes + 64 * rank) >> 4;
          umma_bf16_ss(dS, dQR + rq, dK + rk, idesc_qk, 1u);
          umma_bf16_ss(dS, dQR + rq + 2, dK + rk + 2, idesc_qk, 1u);
        }
        mma_issued_any = true;
        MLA_TRACE_AT(g < 512, 4096 + 4 * g + 1);
        umma_commit(&bars->sfull[g & 1]);
        if (qk.last()) umma_commit(&bars->qempty);
      }
    }
  } else if (warp == C::kPvWarp) {
    // ------------------------------------------------------------ PV issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
      // A = P [128 x 64 tokens], K-major; B = V [64 tokens x 256], MN-major with
      // N blocks of 64 columns = the 4 latent boxes, 8 KB apart.
      const uint64_t dP0 = C::kPSw64 ? smem_desc_sw64(smem_u32(smem + C::kOffP), 16, 512)
                                     : smem_desc_sw128(smem_u32(smem + C::kOffP), 16, 1024);
      const uint64_t dV = smem_desc_sw128(smem_u32(smem + C::kOffKV), kKvBoxBytes, 1024);
      TileIter pv{SegIter{seq, p.batch, x0, x1, b_first}};
      pv.start();
      for (int g = 0; pv.valid; pv.advance(), ++g) {
        const int pb = g % C::kPBufs;
        if (!mbar_wait(&bars->pfull[pb], (g / C::kPBufs) & 1, tmo, abort_flag)) break;
        tc_fence_after();
        MLA_TRACE_AT(g < 512, 4096 + 4 * g + 2);
        MLA_TL(g == 0, 7);
        MLA_TL(true, 14);
        const uint64_t dP = dP0 + static_cast<uint64_t>(((pb % C::kPSmem) * C::kPBytes) >> 4);
        const uint64_t dVs = dV + static_cast<uint64_t>(((g % kStages) * kStageBytes) >> 4);
        const uint32_t first = pv.first() ? 1u : 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // K-step k: tokens 16k..16k+15 of P
          const uint32_t aoff = C::kPSw64 ? static_cast<uint32_t>((k >> 1) * kRows * 64 + (k & 1) * 32)
                                          : static_cast<uint32_t>(k * 32);
          umma_bf16_ss(tmem + kTmemO, dP + static_cast<uint64_t>(aoff >> 4),
                       dVs + static_cast<uint64_t>((k * 2048) >> 4), idesc_pv, (k == 0 && first) ? 0u : 1u);
        }
        pv_issued_any = true;
        MLA_TRACE_AT(g < 512, 4096 + 4 * g + 3);
        mbar_arrive(&bars->pvissued[g & 3]);
        umma_commit(&bars->empty[g % kStages]);
        if constexpr (C::kPair)
          umma_commit_cluster(&bars->pvdone[g & 1], 0x3);   // both CTAs: P is free once both PVs are done
        else
          umma_commit(&bars->pvdone[pb]);
      }
    }
  } else if (C::is_xchg(warp)) {
    // ------------------------------------------------------------ exchange warps (pair path)
    // Warp q4 handles rows 32*q4..+31 of the tiles whose softmax the peer owns
    // (g % 2 != rank): it sends this CTA's partial S (both 32-token halves,
    // 4 KB each, TMEM -> registers -> staging -> one bulk shared::cluster copy
    // per half), zeroes the V tail of this CTA's stage, takes the tile's
    // running max m_g from the peer, rescales this CTA's O rows when m_g grew,
    // and lets the PV issuer go once the peer's P rows have landed.
    if constexpr (C::kPair) {
      const int q4 = warp & 3;
      const int row = q4 * 32 + lane;
      const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
      const uint32_t sX = smem_u32(smem + C::kOffX);
      const uint32_t sXS = smem_u32(smem + C::kOffXS);
      float* red = reinterpret_cast<float*>(smem + C::kOffRed);
      float* mloc = red + 6 * kRows;   // [2][kRows] m of the latest tiles (by tile parity)
      float* mh = red + 8 * kRows;     // [2][kRows] m from the peer (by owned-tile parity of the peer)
      TileIter xt{SegIter{seq, p.batch, x0, x1, b_first}};
      xt.start();
      int L = 0, n_pages = 0;
      for (int g = 0; xt.valid; xt.advance(), ++g) {
        if (xt.first()) {
          const int32_t* sq = seq + static_cast<size_t>(xt.b) * kSeqWords;
          L = sq[kSeqLen];
          n_pages = sq[kSeqPages];
        }
        if (static_cast<uint32_t>(g & 1) == rank) continue;   // this CTA's softmax warps own it
        [[maybe_unused]] const bool tx = (warp == C::kXchgWarp0 && lane == 0 && g < 128);
        MLA_TRACE_AT(tx, 2048 + 16 * g + 0);
        // ---- this CTA's partial S of the peer's tile -> the peer
        if (!mbar_wait(&bars->sfull[g & 1], (g >> 1) & 1, tmo, abort_flag)) break;
        tc_fence_after();
        float a[32], c[32];
        tmem_ld32(tmem + lane_base + kTmemS + 64u * (g & 1), a);
        tmem_ld32(tmem + lane_base + kTmemS + 64u * (g & 1) + 32u, c);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->sfree[g & 1]);
        // two 4 KB halves through this quarter's staging slice, in the receiver's X layout
        const uint32_t stg = sXS + static_cast<uint32_t>(q4 * 4096 + lane * 128);
        bool sent = true;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (lane == 0) bulk_wait_read_all();   // the previous send has read the staging slice
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float* v = h == 0 ? &a[4 * j] : &c[4 * j];
            st_shared_v4_u32(stg + static_cast<uint32_t>((j ^ (lane & 7)) << 4), __float_as_uint(v[0]),
                             __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            // the peer's softmax warp (q4, h) has consumed the previous tile it owns
            if (g >= 2 && !mbar_wait<true>(&bars->xempty[0][q4][h], ((g >> 1) - 1) & 1, tmo, abort_flag)) {
              sent = false;
            } else {
              bulk_copy_to_peer(mapa_shared(sX + static_cast<uint32_t>(h * kRows * 128 + q4 * 4096), peer),
                                sXS + static_cast<uint32_t>(q4 * 4096), 32 * 128,
                                mapa_shared(smem_u32(&bars->xfull[0][q4][h]), peer));
              bulk_commit_group();
            }
          }
          if (__shfl_sync(0xffffffffu, sent ? 1 : 0, 0) == 0) break;
        }
        if (!sent) break;
        MLA_TRACE_AT(tx, 2048 + 16 * g + 1);
        // ---- tail rows of the sequence's last page are not context: zero them in this CTA's V half
        if (xt.i == n_pages - 1 && (L % kPage) != 0) {
          // fp8: the stage was written by the converter warps (their barrier
          // orders those writes before these)
          if (kFp8 && !mbar_wait(&bars->full[g % kStages], (g / kStages) & 1, tmo, abort_flag)) break;
          const int tail = L % kPage;
          uint8_t* vst = smem + C::kOffKV + (g % kStages) * kStageBytes;
          const int per_box = (kPage - tail) * 8;
          for (int idx = row; idx < 4 * per_box; idx += kRows) {
            const int box = idx / per_box;
            const int rem = idx % per_box;
            st_shared_v4_u32(smem_u32(vst + box * kKvBoxBytes + (tail + rem / 8) * 128 + (rem % 8) * 16), 0u, 0u,
                             0u, 0u);
          }
          fence_proxy_async_smem();
        }
        // ---- the tile's running max, sent by the peer early in its softmax
        const int slot = (g >> 1) & 1;
        if (lane == 0) mbar_arrive_expect_tx(&bars->mhfull[slot][q4], 32 * 4);
        if (!mbar_wait<true>(&bars->mhfull[slot][q4], (g >> 2) & 1, tmo, abort_flag)) break;
        MLA_TRACE_AT(tx, 2048 + 16 * g + 2);
        const float m_g = mh[slot * kRows + row];
        float m_prev = -INFINITY;
        if (g >= 1) {   // the previous tile's m, published by this CTA's softmax warps
          if (!mbar_wait(&bars->mready[q4], (g - 1) & 1, tmo, abort_flag)) break;
          if (!xt.first()) m_prev = mloc[((g - 1) & 1) * kRows + row];
        }
        mloc[(g & 1) * kRows + row] = m_g;
        mbar_arrive(&bars->mready[q4]);
        const bool resc = !xt.first() && m_g != m_prev;
        // PV(g-1) done in both CTAs. Waited at every tile of this warp (never
        // costs time: the peer copies P(g) only after it), so that when this
        // warp waits on tile g-1, tile g-3 (same barrier, previous phase) is
        // known to be complete and the parity wait cannot alias.
        if (g >= 1 && !mbar_wait(&bars->pvdone[(g - 1) & 1], ((g - 1) >> 1) & 1, tmo, abort_flag)) break;
        MLA_TRACE_AT(tx, 2048 + 16 * g + 3);
        if (__any_sync(0xffffffffu, resc)) {   // O rows of this quarter, all 256 columns
          tc_fence_after();
          const float al = resc ? ex2_approx(m_prev - m_g) : 1.f;
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            float o[32];
            const uint32_t ta = tmem + lane_base + kTmemO + 32u * cc;
            tmem_ld32(ta, o);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] *= al;
            tmem_st32(ta, o);
          }
          tc_wait_st();
        }
        tc_fence_before();
        // PV may go once these rows are rescaled and the peer's P rows (4 KB) have landed
        if (lane == 0)
          mbar_arrive_expect_tx(&bars->pfull[g & 1], 32 * 128);
        else
          mbar_arrive(&bars->pfull[g & 1]);
        MLA_TRACE_AT(tx, 2048 + 16 * g + 4);
      }
    }
  } else if (warp >= C::kCvtWarp0) {
    // ------------------------------------------------------------ fp8 converters
    if constexpr (kFp8) {
      const int ct = threadIdx.x - C::kCvtWarp0 * 32;   // 0 .. kCvtThreads-1
      TileIter cv{SegIter{seq, p.batch, x0, x1, b_first}};
      cv.start();
      [[maybe_unused]] const bool tc = (ct == 0);   // trace: converter thread 0 (region of softmax warp 1)
      // This thread's chunks of 16 codes, k = 0..9 of every tile: k < 8 are latent
      // chunks (token ct/16 + 8k, column chunk ct%16), k = 8, 9 rope chunks (token
      // ct/4 + 32(k-8), column chunk ct%4). Their byte offsets in the raw stage and
      // in the bf16 stage differ by a constant per k (8 tokens = 1 KB in a 128 B-row
      // box; 32 tokens = 2 KB of 64 B rope rows, 4 KB of bf16 rows), and the second
      // half of a chunk's 16 bf16 values is the neighbouring 16-byte chunk of the
      // same swizzled row: offset ^ 16.
      static_assert(C::kCvtThreads == 128, "the chunk offsets assume 128 converter threads");
      const int lt = ct >> 4, lc = ct & 15, rt = ct >> 2, rc = ct & 3;
      const uint32_t ld_lat = static_cast<uint32_t>((lc >> 3) * kRawLatBytes) + sw128(lt, lc & 7);
      const uint32_t st_lat = static_cast<uint32_t>((lc >> 2) * kKvBoxBytes) + sw128(lt, (lc & 3) * 2);
      const uint32_t ld_rope = static_cast<uint32_t>(kRawRopeOff + rt * 64 + rc * 16);
      const uint32_t st_rope = static_cast<uint32_t>(4 * kKvBoxBytes) + sw128(rt, rc * 2);
      for (int g = 0; cv.valid; cv.advance(), ++g) {
        const int r = g % kRaw, s = g % kStages;
        if (!mbar_wait(&bars->rawfull[r], (g / kRaw) & 1, tmo, abort_flag)) break;
        MLA_TRACE_AT(tc && g < 128, 2048 + 16 * g + 0);
        const uint8_t* raw = smem + C::kOffRaw + r * kRawStageBytes;
        uint8_t* dst = smem + C::kOffKV + s * kStageBytes;
        // 64 tokens x (16 latent + 4 rope) chunks of 16 codes -> 2 bf16 chunks each.
        // The raw stage is usually ready while the bf16 stage is still read by the
        // PV of tile g - kStages: the first kCvtAhead of this thread's chunks are
        // expanded into registers during that wait, the rest after it.
        constexpr int kPer = kPage * 20 / C::kCvtThreads;   // chunks per thread
        static_assert(kPage * 20 % C::kCvtThreads == 0 && C::kCvtThreads >= kPage, "converter split");
        // chunks expanded before the wait (the rest after it): bounded by registers
        constexpr int kAhead = C::kCvtAhead;
        static_assert(kAhead >= 1 && kAhead < kPer, "converter split");
        auto expand = [&](int k, uint32_t (&o)[8]) {
          const uint4 v = *reinterpret_cast<const uint4*>(
              raw + (k < 8 ? ld_lat + static_cast<uint32_t>(k) * 1024u : ld_rope + static_cast<uint32_t>(k - 8) * 2048u));
          if ((e4m3x4_nan_bits(v.x) | e4m3x4_nan_bits(v.y) | e4m3x4_nan_bits(v.z) | e4m3x4_nan_bits(v.w)) == 0u) {
            e4m3x4_to_bf16x4(v.x, o[0], o[1]);
            e4m3x4_to_bf16x4(v.y, o[2], o[3]);
            e4m3x4_to_bf16x4(v.z, o[4], o[5]);
            e4m3x4_to_bf16x4(v.w, o[6], o[7]);
          } else {   // a NaN code: the conversion unit maps it to NaN
            o[0] = e4m3x2_to_bf16x2(static_cast<uint16_t>(v.x));
            o[1] = e4m3x2_to_bf16x2(static_cast<uint16_t>(v.x >> 16));
            o[2] = e4m3x2_to_bf16x2(static_cast<uint16_t>(v.y));
            o[3] = e4m3x2_to_bf16x2(static_cast<uint16_t>(v.y >> 16));
            o[4] = e4m3x2_to_bf16x2(static_cast<uint16_t>(v.z));
            o[5] = e4m3x2_to_bf16x2(static_cast<uint16_t>(v.z >> 16));
            o[6] = e4m3x2_to_bf16x2(static_cast<uint16_t>(v.w));
            o[7] = e4m3x2_to_bf16x2(static_cast<uint16_t>(v.w >> 16));
          }
        };
        const uint32_t dst32 = smem_u32(dst);
        auto store = [&](int k, const uint32_t (&o)[8]) {
          const uint32_t off =
              k < 8 ? st_lat + static_cast<uint32_t>(k) * 1024u : st_rope + static_cast<uint32_t>(k - 8) * 4096u;
          st_shared_v4_u32(dst32 + off, o[0], o[1], o[2], o[3]);
          st_shared_v4_u32(dst32 + (off ^ 16u), o[4], o[5], o[6], o[7]);
        };
        uint32_t ah[kAhead][8];
#pragma unroll
        for (int k = 0; k < kAhead; ++k) expand(k, ah[k]);
        if (g >= kStages && !mbar_wait(&bars->empty[s], ((g / kStages) - 1) & 1, tmo, abort_flag)) break;
        MLA_TRACE_AT(tc && g < 128, 2048 + 16 * g + 1);
#pragma unroll
        for (int k = 0; k < kAhead; ++k) store(k, ah[k]);
#pragma unroll 1
        for (int k = kAhead; k < kPer; ++k) {
          uint32_t o[8];
          expand(k, o);
          store(k, o);
        }
        const float sc = ct < kPage ? reinterpret_cast<const float*>(raw + kRawScaleOff)[ct] : 0.f;
        if (ct < kPage) reinterpret_cast<float*>(dst + kScaleOff)[ct] = sc;
        fence_proxy_async_smem();
        MLA_TRACE_AT(tc && g < 128, 2048 + 16 * g + 2);
        mbar_arrive(&bars->rawempty[r]);
        mbar_arrive(&bars->full[s]);
      }
    }
  } else if (C::is_softmax(warp)) {
    if constexpr (C::kPair) {
    // ------------------------------------------------------------ softmax warps (pair path)
    // This CTA's softmax owns the tiles g with g % 2 == rank. Two warps per lane
    // quarter split such a tile's 64 tokens (warp (q4, hf): rows 32*q4..+31,
    // tokens 32*hf..+31): own partial S from TMEM plus the peer's from the X
    // buffer, the pair's row max, the running max m_g (kept unless it grows by
    // more than 2^8) published here and sent to the peer at once, exp2, O
    // rescale, P into this CTA's P tile and, per warp, one bulk copy of its 2 KB
    // of P into the peer's P tile. Each CTA keeps the row sum of its own tiles;
    // the pair merges them at the segment's epilogue.
    const int q4 = warp & 3;
    const int hf = warp >> 2;
    const bool lead = hf == 0;                  // the pair's warp that talks to the peer
    const int row = q4 * 32 + lane;
    const int cb = 32 * hf;
    const int sti = hf * kRows + row;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t sX = smem_u32(smem + C::kOffX);
    const uint32_t sP = smem_u32(smem + C::kOffP);
    const uint32_t half_off = static_cast<uint32_t>(hf * kRows * 128);
    // this warp's 2 KB of a P tile (tokens 32*hf..+31 of rows 32*q4..+31) and this
    // thread's 64-byte row in it; also the warp's epilogue staging slice
    const uint32_t pwarp = sP + static_cast<uint32_t>(hf * kRows * 64 + q4 * 2048);
    const uint32_t prow = pwarp + static_cast<uint32_t>((lane >> 3) * 512 + (lane & 7) * 64);
    float* red = reinterpret_cast<float*>(smem + C::kOffRed);
    float* red_max = red;               // [2 tiles][2 halves][kRows]
    float* red_l = red + 4 * kRows;     // [2 halves][kRows]
    float* mloc = red + 6 * kRows;      // [2][kRows] m of the latest tiles (by tile parity)
    float* mh = red + 8 * kRows;        // [2][kRows] written by the peer
    float* mhs = red + 10 * kRows;      // [kRows] m staging for the peer
    float* lbuf = red + 11 * kRows;     // [kRows] written by the peer
    float* lst = red + 12 * kRows;      // [kRows] row-sum staging for the peer
    // The two warps of a quarter meet on an mbarrier with a bounded wait (not a
    // named barrier), so that a warp leaving on a timeout cannot strand its partner.
    int pair_phase = 0;
    auto pair_sync = [&]() -> bool {
      mbar_arrive(&bars->pairb[q4]);
      return mbar_wait(&bars->pairb[q4], (pair_phase++) & 1, tmo, abort_flag);
    };
    const float scale_log2 = p.scale_log2;
    [[maybe_unused]] const bool tr = (warp == 0 && lane == 0);
    float* plse = reinterpret_cast<float*>(reinterpret_cast<char*>(p.ws) + w.plse_off);
    float* po = reinterpret_cast<float*>(reinterpret_cast<char*>(p.ws) + w.po_off);

    auto load_q = [&](int b, int seg) -> bool {   // this thread's half of its query row into TMEM
      if (seg > 0 && !mbar_wait(&bars->qempty, (seg - 1) & 1, tmo, abort_flag)) return false;
      const int qrow = r_tile * kRows + row;
      const bool valid = qrow < p.rows;
      const uint4* src = reinterpret_cast<const uint4*>(p.q) +
                         ((static_cast<size_t>(b) * p.rows + (valid ? qrow : 0)) * kDqk + rank * 256 + 128 * hf) / 8;
      tc_fence_after();
      uint32_t v[64];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint4 x = valid ? __ldg(src + j) : make_uint4(0, 0, 0, 0);
        v[4 * j] = x.x;
        v[4 * j + 1] = x.y;
        v[4 * j + 2] = x.z;
        v[4 * j + 3] = x.w;
      }
      // The first segment's query loads are issued: the TMA warp holds its KV
      // loads back until here, so these small loads do not queue behind them.
      if (seg == 0) mbar_arrive(&bars->qissued);
      tmem_st32u(tmem + lane_base + kTmemQ + 64u * hf, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_st32u(tmem + lane_base + kTmemQ + 64u * hf + 32u, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->qtm);
      MLA_TL(warp == 0 && lane == 0 && seg == 0, 5);
      return true;
    };

    TileIter cur{SegIter{seq, p.batch, x0, x1, b_first}};
    cur.start();
    bool ok = true;
    int g = 0;
    int L = 0, n_pages = 0, splits = 0, slot = 0, rg = 0, last_vis = 0;
    float m_w = -INFINITY, l_w = 0.f;   // m of this CTA's latest owned tile in the segment, and its sum
    float m_cur = -INFINITY;            // m of the latest tile this CTA owned
    while (ok && cur.valid) {
      const int b = cur.b, i = cur.i;
      const bool mine = static_cast<uint32_t>(g & 1) == rank;
      if (cur.first()) {
        const int32_t* sq = seq + static_cast<size_t>(b) * kSeqWords;
        L = sq[kSeqLen];
        n_pages = sq[kSeqPages];
        splits = sq[kSeqSplits];
        slot = splits > 1 ? sq[kSeqSlot] + (c_idx - sq[kSeqFirstC]) : 0;
        rg = r_tile * kRows + row;
        last_vis = L - p.q_len + rg / p.heads;     // query t sees tokens j <= L - T + t
        m_w = -INFINITY;
        l_w = 0.f;
        if (!load_q(b, cur.seg)) { ok = false; break; }
        // the peer has finished staging its previous epilogue in its P rows
        if (cur.seg > 0 && !mbar_wait<true>(&bars->epi[q4], (cur.seg - 1) & 1, tmo, abort_flag)) { ok = false; break; }
      }
      if (mine) {
        MLA_TRACE_AT(tr && g < 128, 16 * g + 0);
        // ---- own partial (this warp's 32 tokens), then the peer's, summed
        if (!mbar_wait(&bars->sfull[g & 1], (g >> 1) & 1, tmo, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float s[32];
        tmem_ld32(tmem + lane_base + kTmemS + 64u * (g & 1) + static_cast<uint32_t>(cb), s);
        tc_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->sfree[g & 1]);
        MLA_TRACE_AT(tr && g < 128, 16 * g + 1);
        MLA_TL(warp == 0 && lane == 0 && g == static_cast<int>(rank), 6);
        if (lane == 0) mbar_arrive_expect_tx(&bars->xfull[0][q4][hf], 32 * 128);
        if (!mbar_wait<true>(&bars->xfull[0][q4][hf], (g >> 1) & 1, tmo, abort_flag)) { ok = false; break; }
        MLA_TRACE_AT(tr && g < 128, 16 * g + 2);
        {
          const uint32_t xr = sX + half_off + row * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 v = ld_shared_v4(xr + ((j ^ (row & 7)) << 4));
            s[4 * j] += v.x;
            s[4 * j + 1] += v.y;
            s[4 * j + 2] += v.z;
            s[4 * j + 3] += v.w;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&bars->xempty[0][q4][hf]), peer));

        const int tok0 = i * kPage + cb;
        const bool masked = tok0 + 31 > last_vis;
        // fp8: token scales multiply whole score columns (the dot product is linear)
        const float* sigma =
            reinterpret_cast<const float*>(smem + C::kOffKV + (g % kStages) * kStageBytes + kScaleOff) + cb;
        if constexpr (kFp8) {   // (the converters' scale copy is ordered before this read by the stage barrier)
          if (!mbar_wait(&bars->full[g % kStages], (g / kStages) & 1, tmo, abort_flag)) { ok = false; break; }
#pragma unroll
          for (int j = 0; j < 32; ++j) s[j] *= sigma[j];
        }
        if (masked) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (tok0 + j > last_vis) s[j] = -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(fmaxf(s[k], s[8 + k]), fmaxf(s[16 + k], s[24 + k]));
        const float mhalf =
            fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        const int rb = (g >> 1) & 1;   // red_max buffer of this owned tile
        red_max[(rb * 2 + hf) * kRows + row] = mhalf;
        // ---- the previous tile's running max (whoever handled it published it).
        // Both warps take it BEFORE the pair meeting: the lead publishes this
        // tile's m (the barrier's next phase, and the slot a later tile
        // overwrites) only after the meeting, so neither warp can find the
        // barrier two phases past the one it waits for.
        float m_prev = -INFINITY;
        if (g >= 1) {
          if (!mbar_wait(&bars->mready[q4], (g - 1) & 1, tmo, abort_flag)) { ok = false; break; }
          if (!cur.first()) m_prev = mloc[((g - 1) & 1) * kRows + row];
        }
        if (!pair_sync()) { ok = false; break; }
        const float mt = fmaxf(mhalf, red_max[(rb * 2 + (hf ^ 1)) * kRows + row]) * scale_log2;
        MLA_TRACE_AT(tr && g < 128, 16 * g + 3);
        MLA_TRACE_AT(tr && g < 128, 16 * g + 4);
        // Keep the running max unless it grows by more than 2^8: P stays <= 256.
        const float m_g = mt > m_prev + 8.f ? mt : m_prev;
        const bool resc = !cur.first() && m_g != m_prev;
        if (lead) {
          mloc[(g & 1) * kRows + row] = m_g;
          mbar_arrive(&bars->mready[q4]);
          // m_g to the peer: its O rows are rescaled by it and its next tile starts from it
          if (lane == 0) bulk_wait_read_all();   // the previous copies have read the staging
          __syncwarp();
          mhs[row] = m_g;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int ms = (g >> 1) & 1;
            bulk_copy_to_peer(mapa_shared(smem_u32(mh + ms * kRows + q4 * 32), peer), smem_u32(mhs + q4 * 32), 32 * 4,
                              mapa_shared(smem_u32(&bars->mhfull[ms][q4]), peer));
            bulk_commit_group();
          }
        }
        m_cur = m_g;
        MLA_TRACE_AT(tr && g < 128, 16 * g + 5);
        const float mu = (m_g == -INFINITY) ? 0.f : m_g;
        const float lscale = (m_w == -INFINITY) ? 0.f : ex2_approx(m_w - mu);
        float sum[4];
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 4; ++k) sum[k] = 0.f;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float p0 = ex2_approx(fmaf(s[j], scale_log2, -mu));
          float p1 = ex2_approx(fmaf(s[j + 1], scale_log2, -mu));
          sum[(j >> 1) & 3] += p0 + p1;
          if constexpr (kFp8) {   // V = sigma * codes: fold sigma into P (0 for masked tokens)
            p0 = (masked && tok0 + j > last_vis) ? 0.f : p0 * sigma[j];
            p1 = (masked && tok0 + j + 1 > last_vis) ? 0.f : p1 * sigma[j + 1];
          }
          pk[j >> 1] = pack_bf16x2(p0, p1);
        }
        l_w = l_w * lscale + ((sum[0] + sum[1]) + (sum[2] + sum[3]));
        m_w = m_g;
        MLA_TRACE_AT(tr && g < 128, 16 * g + 6);
        // ---- P tile and O: the previous tile's PV is done in both CTAs (this
        // warp waited on tile g-3 at its previous tile, so the wait cannot alias)
        if (g >= 1 && !mbar_wait(&bars->pvdone[(g - 1) & 1], ((g - 1) >> 1) & 1, tmo, abort_flag)) { ok = false; break; }
        MLA_TRACE_AT(tr && g < 128, 16 * g + 7);
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {   // this warp's half of O's columns
          const float a = resc ? ex2_approx(m_prev - m_g) : 1.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float o[32];
            const uint32_t ta = tmem + lane_base + kTmemO + 128u * hf + 32u * c;
            tmem_ld32(ta, o);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] *= a;
            tmem_st32(ta, o);
          }
          tc_wait_st();
        }
        if (i == n_pages - 1 && (L % kPage) != 0) {   // zero the tail rows of this CTA's V half
          const int tail = L % kPage;
          uint8_t* vst = smem + C::kOffKV + (g % kStages) * kStageBytes;
          const int per_box = (kPage - tail) * 8;
          for (int idx = sti; idx < 4 * per_box; idx += C::kTileThreads) {
            const int box = idx / per_box;
            const int rem = idx % per_box;
            st_shared_v4_u32(smem_u32(vst + box * kKvBoxBytes + (tail + rem / 8) * 128 + (rem % 8) * 16), 0u, 0u,
                             0u, 0u);
          }
        }
        // this warp's 32 rows x 32 tokens of P (64-byte swizzle: 16-byte unit c of
        // a 64-byte row goes to unit c ^ ((row >> 1) & 3)), then its 2 KB to the peer
#pragma unroll
        for (int c = 0; c < 4; ++c)
          st_shared_v4_u32(prow + static_cast<uint32_t>((c ^ ((row >> 1) & 3)) << 4), pk[4 * c], pk[4 * c + 1],
                           pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          bulk_copy_to_peer(mapa_shared(pwarp, peer), pwarp, 2048, mapa_shared(smem_u32(&bars->pfull[g & 1]), peer));
          bulk_commit_group();
        }
        tc_fence_before();
        mbar_arrive(&bars->pfull[g & 1]);
        MLA_TRACE_AT(tr && g < 128, 16 * g + 8);
        MLA_TL(warp == 0 && lane == 0, 8);
      }
      if (cur.last()) {
        // -------------------------------------------------------- epilogue (both CTAs, every segment)
        float m_fin = m_cur;                 // m of the segment's last tile
        if (!mine) {                         // published by this CTA's exchange warp
          if (!mbar_wait(&bars->mready[q4], g & 1, tmo, abort_flag)) { ok = false; break; }
          m_fin = mloc[(g & 1) * kRows + row];
        }
        // this CTA's share of the row sum, on the final max; then the peer's
        red_l[hf * kRows + row] = (m_w == -INFINITY) ? 0.f : l_w * ex2_approx(m_w - m_fin);
        if (!pair_sync()) { ok = false; break; }
        const float c_own = red_l[row] + red_l[kRows + row];   // same order in both warps
        if (lead) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          lst[row] = c_own;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_expect_tx(&bars->lfull[q4], 32 * 4);   // the peer's share, arriving here
            bulk_copy_to_peer(mapa_shared(smem_u32(lbuf + q4 * 32), peer), smem_u32(lst + q4 * 32), 32 * 4,
                              mapa_shared(smem_u32(&bars->lfull[q4]), peer));
            bulk_commit_group();
          }
        }
        if (!mbar_wait<true>(&bars->lfull[q4], cur.seg & 1, tmo, abort_flag)) { ok = false; break; }
        const float lt = c_own + lbuf[row];   // both CTAs add the same two numbers
        MLA_TL(warp == 0 && lane == 0, 9);
        // PV of the last tile done (tile g-2, the previous phase of this barrier,
        // is known complete: waited here at tile g-1, or by this CTA's exchange
        // warp before it published tile g-1's m, which this warp then waited for)
        if (!mbar_wait(&bars->pvdone[g & 1], (g >> 1) & 1, tmo, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const bool valid_row = rg < p.rows;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float lse_nat = lt > 0.f ? (m_fin + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        // Staging: a 2 KB slice of this quarter's P rows: PV of the last tile is
        // done here and in the peer, this pair writes P again only after the
        // next tile's pair barrier, and the peer copies P rows in again only
        // after the epi signal below.
        const uint32_t stg = pwarp;
        const int row0 = r_tile * kRows + q4 * 32;
        const uint32_t tcol = tmem + lane_base + kTmemO + 128u * hf;
        pdl_wait();   // a self-planned launch stores only once the kernels before it on the stream are done
        if (splits <= 1) {
          char* dst0 = reinterpret_cast<char*>(p.out + (static_cast<size_t>(b) * p.rows + row0) * kDv + rank * 256 + 128 * hf);
          store_o_rows<true, 64>(tcol, stg, lane, inv, dst0, min(32, p.rows - row0));
          if (valid_row && rank == 0 && hf == 0) p.lse[static_cast<size_t>(b) * p.rows + rg] = lse_nat;
        } else {
          const size_t pidx0 = (static_cast<size_t>(slot) * p.row_tiles + r_tile) * kRowsPerTile + q4 * 32;
          store_o_rows<false, 64>(tcol, stg, lane, inv, reinterpret_cast<char*>(po + pidx0 * kDv + rank * 256 + 128 * hf), 32);
          if (rank == 0 && hf == 0) plse[pidx0 + lane] = lse_nat;
        }
        tc_fence_before();
        if (!pair_sync()) { ok = false; break; }   // both warps are done with the staging slices
        if (lead && lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&bars->epi[q4]), peer));
        MLA_TL(warp == 0 && lane == 0, 10);
      }
      cur.advance();
      ++g;
    }
    } else if constexpr (C::kPingPong) {
    // ------------------------------------------------------------ softmax warps (ping-pong)
    // The two warps of lane quarter q4 take alternate tiles: warp (q4, wp) owns
    // rows 32*q4..+31 of tiles g with g % 2 == wp. The running max is handed from
    // one tile's warp to the next through shared memory (mready); each warp keeps
    // the softmax sum of its own tiles, and the pair merges them at the epilogue.
    const int q4 = warp & 3;                    // TMEM lane quarter
    const int wp = warp >> 2;                   // tile parity this warp processes
    const int row = q4 * 32 + lane;             // row within the tile
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t sX = smem_u32(smem + C::kOffX);
    const uint32_t sXS = smem_u32(smem + C::kOffXS);
    float* mbuf = reinterpret_cast<float*>(smem + C::kOffRed);   // [kRows] running max handoff
    float* lbuf = mbuf + kRows;                                   // [2][kRows] epilogue: sum per warp
    float* mlast = lbuf + 2 * kRows;                              // [2][kRows] epilogue: max per warp
    // the quarter's two warps meet on a bounded mbarrier wait (a warp that gives
    // up on a timeout cannot strand its partner)
    int pair_phase = 0;
    auto pair_sync = [&]() -> bool {
      mbar_arrive(&bars->pairb[q4]);
      return mbar_wait(&bars->pairb[q4], (pair_phase++) & 1, tmo, abort_flag);
    };
    const float scale_log2 = p.scale_log2;
    float* plse = reinterpret_cast<float*>(reinterpret_cast<char*>(p.ws) + w.plse_off);
    float* po = reinterpret_cast<float*>(reinterpret_cast<char*>(p.ws) + w.po_off);
    [[maybe_unused]] const bool tr = (warp <= 1 && lane == 0);
    [[maybe_unused]] const int trw = warp * 2048;

    // All 256 latent query columns of this thread's row into TMEM (segment start).
    auto load_q_full = [&](int b, int seg) -> bool {
      if (seg > 0 && !mbar_wait(&bars->qempty, (seg - 1) & 1, tmo, abort_flag)) return false;
      const int qrow = r_tile * kRows + row;
      const bool valid = qrow < p.rows;
      const uint4* src = reinterpret_cast<const uint4*>(p.q) +
                         ((static_cast<size_t>(b) * p.rows + (valid ? qrow : 0)) * kDqk + rank * 256) / 8;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[64];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint4 x = valid ? __ldg(src + h * 16 + j) : make_uint4(0, 0, 0, 0);
          v[4 * j] = x.x;
          v[4 * j + 1] = x.y;
          v[4 * j + 2] = x.z;
          v[4 * j + 3] = x.w;
        }
        tmem_st32u(tmem + lane_base + kTmemQ + 64u * h, *reinterpret_cast<uint32_t(*)[32]>(v));
        tmem_st32u(tmem + lane_base + kTmemQ + 64u * h + 32u, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->qtm);
      MLA_TL(warp == 0 && lane == 0 && seg == 0, 5);
      return true;
    };

    TileIter cur{SegIter{seq, p.batch, x0, x1, b_first}};
    cur.start();
    bool ok = true;
    int g = 0;
    int L = 0, n_pages = 0, splits = 0, slot = 0, rg = 0, last_vis = 0;
    float m_w = -INFINITY, l_w = 0.f;   // max this warp last used, and the sum of its tiles (relative to it)
    while (ok && cur.valid) {
      const int b = cur.b, i = cur.i;
      const bool mine = (g & 1) == wp;
      if (cur.first()) {
        const int32_t* sq = seq + static_cast<size_t>(b) * kSeqWords;
        L = sq[kSeqLen];
        n_pages = sq[kSeqPages];
        splits = sq[kSeqSplits];
        slot = splits > 1 ? sq[kSeqSlot] + (c_idx - sq[kSeqFirstC]) : 0;
        rg = r_tile * kRows + row;
        last_vis = L - p.q_len + rg / p.heads;     // query t sees tokens j <= L - T + t
        m_w = -INFINITY;
        l_w = 0.f;
        if (mine && !load_q_full(b, cur.seg)) { ok = false; break; }
      }
      if (mine) {
        const int xb = g & 1;                      // exchange, staging and P buffers of this tile
        MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 0);
        // ---- own partial S: TMEM -> registers (S buffer freed) -> staging -> peer
        if (!mbar_wait(&bars->sfull[g & 1], (g >> 1) & 1, tmo, abort_flag)) { ok = false; break; }
        MLA_TL(warp == 0 && lane == 0 && g == 0, 6);
        tc_fence_after();
        float s[64];
        {
          float a[32], c[32];
          const uint32_t ta = tmem + lane_base + kTmemS + 64u * (g & 1);
          tmem_ld32(ta, a);
          tmem_ld32(ta + 32, c);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            s[j] = a[j];
            s[32 + j] = c[j];
          }
        }
        tc_fence_before();
        mbar_arrive(&bars->sfree[g & 1]);
        MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 1);
        {
          const uint32_t stg = sXS + xb * C::kXBytes + row * 256;
          if (lane == 0) bulk_wait_read_all();   // this warp's previous send from this buffer has been read
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            st_shared_v4_u32(stg + ((j ^ (row & 15)) << 4), __float_as_uint(s[4 * j]), __float_as_uint(s[4 * j + 1]),
                             __float_as_uint(s[4 * j + 2]), __float_as_uint(s[4 * j + 3]));
          fence_proxy_async_smem();
          __syncwarp();
          bool sent = true;
          if (lane == 0) {
            if (g >= 2 && !mbar_wait<true>(&bars->xempty[xb][q4][0], ((g >> 1) - 1) & 1, tmo, abort_flag)) {
              sent = false;
            } else {
              const uint32_t slice = static_cast<uint32_t>(q4 * 32 * 256);
              bulk_copy_to_peer(mapa_shared(sX + xb * C::kXBytes + slice, peer), sXS + xb * C::kXBytes + slice,
                                32 * 256, mapa_shared(smem_u32(&bars->xfull[xb][q4][0]), peer));
              bulk_commit_group();
            }
          }
          if (__shfl_sync(0xffffffffu, sent ? 1 : 0, 0) == 0) { ok = false; break; }
        }
        MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 2);
        // ---- the peer's partial
        if (lane == 0) mbar_arrive_expect_tx(&bars->xfull[xb][q4][0], 32 * 256);
        if (!mbar_wait<true>(&bars->xfull[xb][q4][0], (g >> 1) & 1, tmo, abort_flag)) { ok = false; break; }
        MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 3);
        {
          const uint32_t xr = sX + xb * C::kXBytes + row * 256;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float4 v = ld_shared_v4(xr + ((j ^ (row & 15)) << 4));
            s[4 * j] += v.x;
            s[4 * j + 1] += v.y;
            s[4 * j + 2] += v.z;
            s[4 * j + 3] += v.w;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&bars->xempty[xb][q4][0]), peer));
        MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 4);

        const int tok0 = i * kPage;
        const bool masked = tok0 + kPage - 1 > last_vis;
        const float* sigma = reinterpret_cast<const float*>(smem + C::kOffKV + (g % kStages) * kStageBytes + kScaleOff);
        if constexpr (kFp8) {   // token scales multiply whole score columns (the dot product is linear)
          if (!mbar_wait(&bars->full[g % kStages], (g / kStages) & 1, tmo, abort_flag)) { ok = false; break; }
#pragma unroll
          for (int j = 0; j < 64; ++j) s[j] *= sigma[j];
        }
        if (masked) {
#pragma unroll
          for (int j = 0; j < 64; ++j)
            if (tok0 + j > last_vis) s[j] = -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(s[k], s[8 + k]);
#pragma unroll
        for (int j = 16; j < 64; j += 8)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmaxf(mx[k], s[j + k]);
        const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * scale_log2;
        // ---- running max: take the previous tile's from the other warp, hand ours on
        float m_prev = -INFINITY;
        if (!cur.first()) {
          if (!mbar_wait(&bars->mready[q4], (g - 1) & 1, tmo, abort_flag)) { ok = false; break; }
          m_prev = mbuf[row];
        }
        float m_g = m_prev;
        bool resc = false;
        // Keep the running max unless it grows by more than 2^8: P stays <= 256.
        if (mt > m_prev + 8.f) {
          m_g = mt;
          resc = !cur.first();
        }
        mbuf[row] = m_g;
        mbar_arrive(&bars->mready[q4]);
        MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 5);
        const float mu = (m_g == -INFINITY) ? 0.f : m_g;
        const float lscale = (m_w == -INFINITY) ? 0.f : ex2_approx(m_w - mu);   // this warp's sum onto m_g
        float sum[8];
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) sum[k] = 0.f;
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          float p0 = ex2_approx(fmaf(s[j], scale_log2, -mu));
          float p1 = ex2_approx(fmaf(s[j + 1], scale_log2, -mu));
          sum[(j >> 1) & 7] += p0 + p1;
          if constexpr (kFp8) {   // V = sigma * codes: fold sigma into P (0 for masked tokens)
            p0 = (masked && tok0 + j > last_vis) ? 0.f : p0 * sigma[j];
            p1 = (masked && tok0 + j + 1 > last_vis) ? 0.f : p1 * sigma[j + 1];
          }
          pk[j >> 1] = pack_bf16x2(p0, p1);
        }
        l_w = l_w * lscale + (((sum[0] + sum[1]) + (sum[2] + sum[3])) + ((sum[4] + sum[5]) + (sum[6] + sum[7])));
        m_w = m_g;
        MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 6);
        // ---- P buffer free (PV(g-2) done); O rescale needs PV(g-1) done
        if (g >= 2 && !mbar_wait(&bars->pvdone[xb], ((g >> 1) - 1) & 1, tmo, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
          if (!mbar_wait(&bars->pvdone[xb ^ 1], ((g - 1) >> 1) & 1, tmo, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const float a = resc ? ex2_approx(m_prev - m_g) : 1.f;
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            float o[32];
            const uint32_t ta = tmem + lane_base + kTmemO + 32u * c;
            tmem_ld32(ta, o);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] *= a;
            tmem_st32(ta, o);
          }
          tc_wait_st();
        }
        MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 7);
        if (i == n_pages - 1 && (L % kPage) != 0) {   // zero the tail rows of this CTA's V half
          const int tail = L % kPage;
          uint8_t* vst = smem + C::kOffKV + (g % kStages) * kStageBytes;
          const int per_box = (kPage - tail) * 8;
          for (int idx = row; idx < 4 * per_box; idx += kRows) {
            const int box = idx / per_box;
            const int rem = idx % per_box;
            st_shared_v4_u32(smem_u32(vst + box * kKvBoxBytes + (tail + rem / 8) * 128 + (rem % 8) * 16), 0u, 0u,
                             0u, 0u);
          }
        }
        const uint32_t prow = smem_u32(smem + C::kOffP + xb * C::kPBytes) + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_shared_v4_u32(prow + ((c ^ (row & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->pfull[xb]);
        MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 8);
        MLA_TL(lane == 0 && cur.last(), 8);
      }
      if (cur.last()) {
        // -------------------------------------------------------- epilogue (both warps)
        lbuf[wp * kRows + row] = l_w;
        mlast[wp * kRows + row] = m_w;
        if (!pair_sync()) { ok = false; break; }
        const float mA = mlast[row], mB = mlast[kRows + row];
        const float lA = lbuf[row], lB = lbuf[kRows + row];
        if (!pair_sync()) { ok = false; break; }   // both have read before either writes again
        const float m_fin = fmaxf(mA, mB);   // the last tile's max (the running max only grows)
        const float mf = (m_fin == -INFINITY) ? 0.f : m_fin;
        const float lt = (mA == -INFINITY ? 0.f : lA * ex2_approx(mA - mf)) + (mB == -INFINITY ? 0.f : lB * ex2_approx(mB - mf));
        if (!mbar_wait(&bars->pvdone[g & 1], (g >> 1) & 1, tmo, abort_flag)) { ok = false; break; }
        MLA_TL(warp == 0 && lane == 0, 9);
        tc_fence_after();
        const bool valid_row = rg < p.rows;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float lse_nat = lt > 0.f ? (m_fin + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        // staging: this warp's own exchange staging slice, once its last send has been read
        const uint32_t stg = sXS + wp * C::kXBytes + q4 * 32 * 256;
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
        const int row0 = r_tile * kRows + q4 * 32;   // this warp's first query row
        const uint32_t tcol = tmem + lane_base + kTmemO + 128u * wp;
        pdl_wait();   // a self-planned launch stores only once the kernels before it on the stream are done
        if (splits <= 1) {
          char* dst0 = reinterpret_cast<char*>(p.out + (static_cast<size_t>(b) * p.rows + row0) * kDv + rank * 256 + 128 * wp);
          store_o_rows<true, 128>(tcol, stg, lane, inv, dst0, min(32, p.rows - row0));
          if (valid_row && rank == 0 && wp == 0) p.lse[static_cast<size_t>(b) * p.rows + rg] = lse_nat;
        } else {
          const size_t pidx0 = (static_cast<size_t>(slot) * p.row_tiles + r_tile) * kRowsPerTile + q4 * 32;
          store_o_rows<false, 128>(tcol, stg, lane, inv, reinterpret_cast<char*>(po + pidx0 * kDv + rank * 256 + 128 * wp), 32);
          if (rank == 0 && wp == 0) plse[pidx0 + lane] = lse_nat;
        }
        MLA_TL(warp == 0 && lane == 0, 10);
        tc_fence_before();
      }
      cur.advance();
      ++g;
    }
    } else {
    // ------------------------------------------------------------ softmax warps
    // Two warps per lane quarter: warp (q4, hf) owns rows 32*q4..+31 and tokens
    // 32*hf..+31 of every tile; the pair agrees on each tile's row max through
    // shared memory and a bounded mbarrier meeting, and splits O's 256 columns
    // in halves. One exchange buffer: tile g's partial S is sent at its start.
    static_assert(C::kXBufs == 1, "the split path uses one exchange buffer");
    const int q4 = warp & 3;                    // TMEM lane quarter
    const int hf = warp >> 2;                   // token half of the tile this warp owns
    const int row = q4 * 32 + lane;             // row within the tile
    const int cb = 32 * hf;                     // first token (column) of this warp's half
    const int sti = hf * kRows + row;           // index among the softmax threads
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t sX = smem_u32(smem + C::kOffX);
    const uint32_t sXS = smem_u32(smem + C::kOffXS);
    const uint32_t half_off = static_cast<uint32_t>(hf * kRows * 128);   // this half's slice of X / staging
    const uint32_t prow = smem_u32(smem + C::kOffP) + (row >> 3) * 1024 + (row & 7) * 128;
    float* red_max = reinterpret_cast<float*>(smem + C::kOffRed);          // [2 tiles][2 halves][kRows]
    float* red_l = red_max + 4 * kRows;                                     // [2 halves][kRows]
    // the quarter's two warps meet on a bounded mbarrier wait (a warp that gives
    // up on a timeout cannot strand its partner)
    int pair_phase = 0;
    auto pair_sync = [&]() -> bool {
      mbar_arrive(&bars->pairb[q4]);
      return mbar_wait(&bars->pairb[q4], (pair_phase++) & 1, tmo, abort_flag);
    };
    const float scale_log2 = p.scale_log2;
    float* plse = reinterpret_cast<float*>(reinterpret_cast<char*>(p.ws) + w.plse_off);
    float* po = reinterpret_cast<float*>(reinterpret_cast<char*>(p.ws) + w.po_off);
    // (softmax warp 0 only: warp 1's trace region holds the converters' stamps)
    [[maybe_unused]] const bool tr = (warp == 0 && lane == 0);
    [[maybe_unused]] const int trw = 0;

    // Writes this thread's half of its query row (128 of this CTA's 256 latent
    // columns) into TMEM for the segment of sequence b, once the previous
    // segment's QKs are done.
    auto load_q = [&](int b, int seg) -> bool {
      if (seg > 0 && !mbar_wait(&bars->qempty, (seg - 1) & 1, tmo, abort_flag)) return false;
      const int qrow = r_tile * kRows + row;
      const bool valid = qrow < p.rows;
      const uint4* src = reinterpret_cast<const uint4*>(p.q) +
                         ((static_cast<size_t>(b) * p.rows + (valid ? qrow : 0)) * kDqk + rank * 256 + 128 * hf) / 8;
      tc_fence_after();
      uint32_t v[64];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint4 x = valid ? __ldg(src + j) : make_uint4(0, 0, 0, 0);
        v[4 * j] = x.x;
        v[4 * j + 1] = x.y;
        v[4 * j + 2] = x.z;
        v[4 * j + 3] = x.w;
      }
      tmem_st32u(tmem + lane_base + kTmemQ + 64u * hf, *reinterpret_cast<uint32_t(*)[32]>(v));
      tmem_st32u(tmem + lane_base + kTmemQ + 64u * hf + 32u, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->qtm);
      return true;
    };
    // Loads this warp's 32 columns of this thread's row of tile h's partial S.
    auto load_s = [&](int h, float (&s)[32]) {
      tmem_ld32(tmem + lane_base + kTmemS + 64u * (h & 1) + static_cast<uint32_t>(cb), s);
      tc_wait_ld();
    };
    // Sends this CTA's partial S (this warp's 32 rows x 32 tokens) of tile h to
    // the peer's X buffer: staged locally in the same swizzled layout, then one
    // lane sends the contiguous 4 KB with a bulk copy counted on the peer's
    // barrier. The own partial stays in s.
    auto send = [&](int h, float (&s)[32], int tb) -> bool {
      if (!mbar_wait(&bars->sfull[h & 1], (h >> 1) & 1, tmo, abort_flag)) return false;
      MLA_TRACE_AT(tr && tb >= 0, trw + tb + 1);
      tc_fence_after();
      load_s(h, s);
      tc_fence_before();
      mbar_arrive(&bars->sfree[h & 1]);
      MLA_TRACE_AT(tr && tb >= 0, trw + tb + 2);
      const uint32_t stg = sXS + half_off + row * 128;
      if (lane == 0) bulk_wait_read_all();   // the previous send has read the staging slice
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_shared_v4_u32(stg + ((j ^ (row & 7)) << 4), __float_as_uint(s[4 * j]), __float_as_uint(s[4 * j + 1]),
                         __float_as_uint(s[4 * j + 2]), __float_as_uint(s[4 * j + 3]));
      MLA_TRACE_AT(tr && tb >= 0, trw + tb + 11);
      fence_proxy_async_smem();
      MLA_TRACE_AT(tr && tb >= 0, trw + tb + 12);
      __syncwarp();
      bool sent = true;
      if (lane == 0) {
        if (h >= 1 && !mbar_wait<true>(&bars->xempty[0][q4][hf], (h - 1) & 1, tmo, abort_flag)) {
          sent = false;
        } else {
          MLA_TRACE_AT(tr && tb >= 0, trw + tb + 3);
          const uint32_t slice = half_off + static_cast<uint32_t>(q4 * 32 * 128);
          bulk_copy_to_peer(mapa_shared(sX + slice, peer), sXS + slice, 32 * 128,
                            mapa_shared(smem_u32(&bars->xfull[0][q4][hf]), peer));
          bulk_commit_group();
        }
      }
      sent = __shfl_sync(0xffffffffu, sent ? 1 : 0, 0) != 0;
      MLA_TRACE_AT(tr && tb >= 0, trw + tb + 4);
      return sent;
    };

    TileIter cur{SegIter{seq, p.batch, x0, x1, b_first}};
    cur.start();
    bool ok = true;
    if (cur.valid) ok = load_q(cur.b, 0);
    int g = 0;
    int L = 0, n_pages = 0, splits = 0, slot = 0, rg = 0, last_vis = 0;
    float m = -INFINITY, l = 0.f;   // running max (both warps of a pair agree) and this half's sum
    while (ok && cur.valid) {
      const int b = cur.b, i = cur.i;
      if (cur.first()) {
        const int32_t* sq = seq + static_cast<size_t>(b) * kSeqWords;
        L = sq[kSeqLen];
        n_pages = sq[kSeqPages];
        splits = sq[kSeqSplits];
        slot = splits > 1 ? sq[kSeqSlot] + (c_idx - sq[kSeqFirstC]) : 0;
        rg = r_tile * kRows + row;                 // query row index (t, h)
        last_vis = L - p.q_len + rg / p.heads;     // query t sees tokens j <= L - T + t
        m = -INFINITY;
        l = 0.f;
        if (cur.seg > 0 && !load_q(b, cur.seg)) { ok = false; break; }
      }
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 0);
      // partial-S exchange: this tile's own partial out to the peer, the peer's in
      float s[32];
      if (!send(g, s, g < 128 ? 16 * g : -1)) { ok = false; break; }
      if (lane == 0) mbar_arrive_expect_tx(&bars->xfull[0][q4][hf], 32 * 128);
      if (!mbar_wait<true>(&bars->xfull[0][q4][hf], g & 1, tmo, abort_flag)) { ok = false; break; }
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 5);
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 6);
      {
        const uint32_t xr = sX + half_off + row * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 v = ld_shared_v4(xr + ((j ^ (row & 7)) << 4));
          s[4 * j] += v.x;
          s[4 * j + 1] += v.y;
          s[4 * j + 2] += v.z;
          s[4 * j + 3] += v.w;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(mapa_shared(smem_u32(&bars->xempty[0][q4][hf]), peer));
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 7);

      const int tok0 = i * kPage + cb;             // first token of this warp's half
      const bool masked = tok0 + 31 > last_vis;
      const float* sigma = reinterpret_cast<const float*>(smem + C::kOffKV + (g % kStages) * kStageBytes + kScaleOff) + cb;
      if constexpr (kFp8) {   // token scales multiply whole score columns (the dot product is linear)
        // (the converters' scale copy is ordered before this read by this stage's barrier)
        if (!mbar_wait(&bars->full[g % kStages], (g / kStages) & 1, tmo, abort_flag)) { ok = false; break; }
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] *= sigma[j];
      }
      // Mask tokens past this query's position; this half's max (tree), then the pair's.
      if (masked) {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (tok0 + j > last_vis) s[j] = -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmaxf(fmaxf(s[k], s[8 + k]), fmaxf(s[16 + k], s[24 + k]));
      const float mh = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      red_max[((g & 1) * 2 + hf) * kRows + row] = mh;
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 13);
      if (!pair_sync()) { ok = false; break; }
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 14);
      const float mt = fmaxf(mh, red_max[((g & 1) * 2 + (hf ^ 1)) * kRows + row]) * scale_log2;
      const float m_new = fmaxf(m, mt);
      float alpha = 1.f;
      bool resc = false;
      // Keep the running max unless it grows by more than 2^8: P stays <= 256.
      if (m_new > m + 8.f) {
        alpha = ex2_approx(m - m_new);
        resc = !cur.first();
        m = m_new;
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      float sum[4];
      uint32_t pk[16];
#pragma unroll
      for (int k = 0; k < 4; ++k) sum[k] = 0.f;
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        float p0 = ex2_approx(fmaf(s[j], scale_log2, -mu));
        float p1 = ex2_approx(fmaf(s[j + 1], scale_log2, -mu));
        sum[(j >> 1) & 3] += p0 + p1;
        if constexpr (kFp8) {   // V = sigma * codes: fold sigma into P (0 for masked tokens)
          p0 = (masked && tok0 + j > last_vis) ? 0.f : p0 * sigma[j];
          p1 = (masked && tok0 + j + 1 > last_vis) ? 0.f : p1 * sigma[j + 1];
        }
        pk[j >> 1] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + ((sum[0] + sum[1]) + (sum[2] + sum[3]));
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 15);

      // PV(g-1) done: P buffer free and O stable.
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 8);
      if (g >= 1 && !mbar_wait(&bars->pvdone[0], (g - 1) & 1, tmo, abort_flag)) { ok = false; break; }
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 9);
      tc_fence_after();
      if (__any_sync(0xffffffffu, resc)) {   // this warp's half of O's columns
        const float a = resc ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          const uint32_t ta = tmem + lane_base + kTmemO + 128u * hf + 32u * c;
          tmem_ld32(ta, o);
          tc_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] *= a;
          tmem_st32(ta, o);
        }
        tc_wait_st();
      }
      // Tail rows of the sequence's last page are not part of the context:
      // zero them in this CTA's V half so stale data (even NaN) cannot leak
      // through 0 * V in the PV product.
      if (i == n_pages - 1 && (L % kPage) != 0) {
        const int tail = L % kPage;
        uint8_t* vst = smem + C::kOffKV + (g % kStages) * kStageBytes;
        const int per_box = (kPage - tail) * 8;        // 16-byte chunks per box
        for (int idx = sti; idx < 4 * per_box; idx += C::kSoftmaxThreads) {
          const int box = idx / per_box;
          const int rem = idx % per_box;
          st_shared_v4_u32(smem_u32(vst + box * kKvBoxBytes + (tail + rem / 8) * 128 + (rem % 8) * 16), 0u, 0u,
                           0u, 0u);
        }
      }
      // this half of the P row -> bf16, 128B-swizzled K-major tile
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t ch = static_cast<uint32_t>((4 * hf + c) ^ (row & 7));
        st_shared_v4_u32(prow + ch * 16, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars->pfull[0]);
      MLA_TRACE_AT(tr && g < 128, trw + 16 * g + 10);

      if (cur.last()) {
        // -------------------------------------------------------- epilogue
        red_l[hf * kRows + row] = l;
        if (!pair_sync()) { ok = false; break; }
        const float lt = red_l[row] + red_l[kRows + row];   // same order in both warps
        if (!mbar_wait(&bars->pvdone[0], g & 1, tmo, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const bool valid_row = rg < p.rows;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const float lse_nat = lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
        // staging: this warp's own exchange staging slice, once its last send has been read
        constexpr int kStgRow = 128;
        const uint32_t stg = sXS + half_off + static_cast<uint32_t>(q4 * 32 * 128);
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
        const int row0 = r_tile * kRows + q4 * 32;   // this warp's first query row
        const uint32_t tcol = tmem + lane_base + kTmemO + 128u * hf;
        pdl_wait();   // a self-planned launch stores only once the kernels before it on the stream are done
        if (splits <= 1) {
          char* dst0 = reinterpret_cast<char*>(p.out + (static_cast<size_t>(b) * p.rows + row0) * kDv + rank * 256 + 128 * hf);
          store_o_rows<true, kStgRow>(tcol, stg, lane, inv, dst0, min(32, p.rows - row0));
          if (valid_row && rank == 0 && hf == 0) p.lse[static_cast<size_t>(b) * p.rows + rg] = lse_nat;
        } else {
          const size_t pidx0 = (static_cast<size_t>(slot) * p.row_tiles + r_tile) * kRowsPerTile + q4 * 32;
          store_o_rows<false, kStgRow>(tcol, stg, lane, inv, reinterpret_cast<char*>(po + pidx0 * kDv + rank * 256 + 128 * hf), 32);
          if (rank == 0 && hf == 0) plse[pidx0 + lane] = lse_nat;
        }
        tc_fence_before();
      }
      cur.advance();
      ++g;
    }
    }  // if constexpr (kPingPong)
  }

  // ---------------------------------------------------------------- teardown
  if ((C::is_softmax(warp) || C::is_xchg(warp)) && lane == 0) bulk_wait_all();   // exchange copies have been read
  __syncthreads();
  MLA_TL(threadIdx.x == 0, 11);
  if (threadIdx.x == 0) {
    // The flag word is cleared by the planner kernel at the start of the step,
    // which a self-planned launch may have run beside: write after it is done.
    pdl_wait();
    int f = bars->flags | (*abort_flag ? kFlagTimeout : 0);
    if (blockIdx.x == 0) {   // the planner's block-table check, if it ran
      const int nchk = min(hdr[kHdrChecks], kMaxCheckCtas);
      for (int k = 0; k < nchk; ++k)
        if (hdr[kHdrCheck0 + k]) f |= kFlagBadPage;
      // the combine kernel follows the planner's plan: it must be the one used here
      if (p.self_plan && (hdr[kHdrClusters] != bars->plan_hdr[0] || hdr[kHdrPayload] != bars->plan_hdr[1] ||
                          hdr[kHdrTotal] != bars->plan_hdr[2]))
        f |= kFlagPlanMismatch;
    }
    if (f) atomicOr(&hdr[kHdrFlag], f);
  }
  if (*abort_flag) {
    // Let every copy and MMA this CTA started land before its memory goes away.
    if (warp == C::kTmaWarp && lane == 0) {
      constexpr int kRing = kFp8 ? kRaw : kStages;
      for (int gg = max(0, tma_last_g - kRing + 1); gg <= tma_last_g; ++gg) {
        volatile int never = 0;
        if (kFp8)
          mbar_wait(&bars->rawfull[gg % kRing], (gg / kRing) & 1, kDrainTimeoutNs, &never);
        else
          mbar_wait(&bars->full[gg % kRing], (gg / kRing) & 1, kDrainTimeoutNs, &never);
      }
      if (tma_q_issued > 0) {
        volatile int never = 0;
        mbar_wait(&bars->qfull, (tma_q_issued - 1) & 1, kDrainTimeoutNs, &never);
      }
    }
    if (warp == C::kQkWarp && lane == 0 && mma_issued_any) {
      umma_commit(&bars->drain_qk);
      volatile int never = 0;
      mbar_wait(&bars->drain_qk, 0, kDrainTimeoutNs, &never);
    }
    if (warp == C::kPvWarp && lane == 0 && pv_issued_any) {
      umma_commit(&bars->drain_pv);
      volatile int never = 0;
      mbar_wait(&bars->drain_pv, 0, kDrainTimeoutNs, &never);
    }
    __syncthreads();
  }
  if (warp == C::kQkWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync_all();  // no CTA leaves while its peer may still touch its shared memory
  MLA_TL(threadIdx.x == 0, 12);
}

template <int kRows, bool kFp8>
cudaLaunchConfig_t launch_config(int clusters, cudaStream_t stream, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(Cfg<kRows, kFp8>::kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg<kRows, kFp8>::kSmemBytes;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cfg;
}

template <int kRows, bool kFp8>
cudaError_t max_clusters(int* clusters) {
  cudaError_t e = cudaFuncSetAttribute(mla_decode_kernel<kRows, kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<kRows, kFp8>::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = launch_config<kRows, kFp8>(1024, nullptr, attr);
  cfg.numAttrs = 1;  // occupancy query: cluster shape only
  return cudaOccupancyMaxActiveClusters(clusters, mla_decode_kernel<kRows, kFp8>, &cfg);
}

template <int kRows, bool kFp8>
cudaError_t launch(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const CUtensorMap& tm_kv2,
                   const DecodeParams& p, cudaStream_t stream) {
  cudaLaunchAttribute attr[2];
  cudaLaunchConfig_t cfg = launch_config<kRows, kFp8>(p.row_tiles * p.c_max, stream, attr);
  return cudaLaunchKernelEx(&cfg, mla_decode_kernel<kRows, kFp8>, tm_q, tm_kv, tm_kv2, p);
}

}  // namespace

cudaError_t launch_decode(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const CUtensorMap& tm_kv2,
                          const DecodeParams& p, cudaStream_t stream) {
  // The dynamic shared-memory limit was raised for this device by
  // decode_max_active_clusters(), which the host API calls first.
  if (p.fp8) {
    return p.tile_rows == 64 ? launch<64, true>(tm_q, tm_kv, tm_kv2, p, stream)
                             : launch<128, true>(tm_q, tm_kv, tm_kv2, p, stream);
  }
  return p.tile_rows == 64 ? launch<64, false>(tm_q, tm_kv, tm_kv2, p, stream)
                           : launch<128, false>(tm_q, tm_kv, tm_kv2, p, stream);
}

cudaError_t decode_max_active_clusters(int tile_rows, bool fp8, int* clusters) {
  if (fp8) return tile_rows == 64 ? max_clusters<64, true>(clusters) : max_clusters<128, true>(clusters);
  return tile_rows == 64 ? max_clusters<64, false>(clusters) : max_clusters<128, false>(clusters);
}

}  // namespace mla
