// K1: MLA decode main kernel for a bf16 paged latent cache (sm_100a).
//
// Work unit: one cluster of two CTAs owns a contiguous range of (sequence,
// page) work from the planner (K0) for one 128-row tile of query rows (t, h).
// The pair splits the work so that neither CTA duplicates tensor-core flops
// and both fit their accumulators in tensor memory:
//
//   * PV is split along V's 512 columns: CTA r accumulates O[:, 256r:256r+256]
//     (128 lanes x 256 fp32 columns of TMEM).
//   * QK^T is split along the 576-wide contraction: CTA r contracts latent
//     columns [256r, 256r+256) - the same columns it needs as its V half - plus
//     rope columns [512+32r, 512+32r+32). The two partial score tiles are summed
//     through distributed shared memory, so both CTAs hold the same S and take
//     bit-identical softmax decisions.
//
// Per 64-token page (one KV tile) and CTA:
//   TMA warp  : block_table[b, i] -> 5 boxes (4 latent + rope) of 64x64 bf16,
//               128B-swizzled, into a ring stage;
//   MMA thread: S_r = Q_r K_r^T (18 x tcgen05.mma M128 N64 K16) into TMEM;
//               then O_r += P V_r (4 x tcgen05.mma M128 N256 K16);
//   4 softmax warps (one query row per thread): S from TMEM, partial-S
//               exchange with the peer CTA, causal mask among the q_len draft
//               tokens, online softmax in the log2 domain, P (bf16) to shared
//               memory; rare O rescales in TMEM; epilogue O/l (bf16 out, or fp32
//               partial for split sequences) and lse.
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

constexpr int kThreads = 192;                     // warp0 TMA, warp1 MMA, warps2-5 softmax
constexpr int kStages = 2;
constexpr int kBoxes = 5;                         // 4 latent boxes + 1 rope box
constexpr int kKvBoxBytes = kPage * 128;          // 64 tokens x 64 bf16
constexpr int kStageBytes = kBoxes * kKvBoxBytes; // 40 KB
constexpr int kQBoxBytes = kRowsPerTile * 128;    // 128 rows x 64 bf16
constexpr int kQBytes = kBoxes * kQBoxBytes;      // 80 KB
constexpr int kPBytes = kRowsPerTile * kPage * 2; // P tile, bf16
constexpr int kXBytes = kRowsPerTile * kPage * 4; // partial-S exchange tile, fp32
constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kQBytes;
constexpr int kOffP = kOffKV + kStages * kStageBytes;
constexpr int kOffX = kOffP + kPBytes;
constexpr int kOffBar = kOffX + kXBytes;
constexpr int kSmemBytes = kOffBar + 1024 + 1024;  // barriers + 1 KB alignment slack

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;      // O half: columns [0, 256)
constexpr uint32_t kTmemS = 256;    // S double buffer: [256, 320), [320, 384)

constexpr unsigned long long kDrainTimeoutNs = 200ull * 1000 * 1000;

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t qfull, qempty;
  uint64_t sfull[2], sfree[2];
  uint64_t pfull, pvdone;
  uint64_t xfull[4], xempty[4];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

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

__device__ __forceinline__ int latent_col(int rank, int box) { return box < 4 ? rank * 256 + box * 64 : 512; }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
    mla_decode_bf16_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                           const DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cluster = blockIdx.x >> 1;
  const int r_tile = cluster / p.c_max;
  const int c_idx = cluster % p.c_max;

  const WsLayout w = ws_layout(p.batch, p.row_tiles, p.c_max);
  int32_t* hdr = p.ws;
  const int32_t* seq = reinterpret_cast<const int32_t*>(reinterpret_cast<const char*>(p.ws) + w.seq_off);
  const int32_t* first_b = reinterpret_cast<const int32_t*>(reinterpret_cast<const char*>(p.ws) + w.first_b_off);
  const int clusters = hdr[kHdrClusters];
  // Both CTAs of a cluster take the same branch, so no cluster barrier is skipped.
  if (c_idx >= clusters || r_tile >= p.row_tiles) return;
  const int payload = hdr[kHdrPayload];
  const int x0 = c_idx * payload;
  const int x1 = min(x0 + payload, hdr[kHdrTotal]);
  const int b_first = first_b[c_idx];

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->qfull, 1);
    mbar_init(&bars->qempty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->sfull[i], 1);
      mbar_init(&bars->sfree[i], 128);
    }
    mbar_init(&bars->pfull, 128);
    mbar_init(&bars->pvdone, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&bars->xfull[i], 32);
      mbar_init(&bars->xempty[i], 32);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_kv);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // the peer's barriers are initialised before any remote arrive
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort;
  const unsigned long long tmo = p.timeout_ns;

  // Outstanding-work trackers for the abort drain.
  int tma_last_g = -1, tma_q_issued = 0;
  bool mma_issued_any = false;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      SegIter it{seq, p.batch, x0, x1, b_first};
      int g = 0, segi = 0, b, lo, hi;
      bool ok = true;
      while (ok && it.next(b, lo, hi)) {
        if (segi > 0 && !mbar_wait(&bars->qempty, (segi - 1) & 1, tmo, abort_flag)) break;
        mbar_arrive_expect_tx(&bars->qfull, kQBytes);
        const int row0 = b * p.rows + r_tile * kRowsPerTile;
#pragma unroll
        for (int k = 0; k < kBoxes; ++k)
          tma_load_2d(smem + kOffQ + k * kQBoxBytes, &tm_q, &bars->qfull, latent_col(rank, k), row0);
        tma_q_issued = segi + 1;
        const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_pages;
        for (int i = lo; i < hi; ++i, ++g) {
          const int s = g % kStages;
          if (g >= kStages && !mbar_wait(&bars->empty[s], ((g / kStages) - 1) & 1, tmo, abort_flag)) {
            ok = false;
            break;
          }
          int phys = bt[i];
          if (phys < 0 || phys >= p.num_pages) {
            atomicOr(&hdr[kHdrFlag], kFlagBadPage);
            phys = 0;
          }
          mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
          uint8_t* dst = smem + kOffKV + s * kStageBytes;
#pragma unroll
          for (int k = 0; k < kBoxes; ++k)
            tma_load_3d(dst + k * kKvBoxBytes, &tm_kv, &bars->full[s], latent_col(rank, k), 0, phys);
          tma_last_g = g;
        }
        ++segi;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, false, true);
      const uint32_t sQ = smem_u32(smem + kOffQ);
      const uint32_t sKV = smem_u32(smem + kOffKV);
      const uint32_t sP = smem_u32(smem + kOffP);
      SegIter it{seq, p.batch, x0, x1, b_first};
      int g = 0, segi = 0, b, lo, hi;
      int pending = -1;
      bool pending_first = false;
      bool ok = true;
      auto issue_pv = [&](int h, bool first) -> bool {
        if (!mbar_wait(&bars->pfull, h & 1, tmo, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vbase = sKV + (h % kStages) * kStageBytes;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // A = P [128 x 64 tokens], K-major; B = V [64 tokens x 256], MN-major
          // (N blocks of 64 columns = the 4 latent boxes, 8 KB apart).
          const uint64_t ad = smem_desc_sw128(sP + k * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(vbase + k * 2048, kKvBoxBytes, 1024);
          umma_bf16_ss(tmem + kTmemO, ad, bd, idesc_pv, (first && k == 0) ? 0u : 1u);
        }
        umma_commit(&bars->empty[h % kStages]);
        umma_commit(&bars->pvdone);
        return true;
      };
      while (ok && it.next(b, lo, hi)) {
        if (!mbar_wait(&bars->qfull, segi & 1, tmo, abort_flag)) break;
        tc_fence_after();
        for (int i = lo; i < hi; ++i, ++g) {
          const int s = g % kStages;
          if (!mbar_wait(&bars->full[s], (g / kStages) & 1, tmo, abort_flag)) { ok = false; break; }
          if (g >= 2 && !mbar_wait(&bars->sfree[g & 1], ((g >> 1) - 1) & 1, tmo, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kvb = sKV + s * kStageBytes;
          const uint32_t dS = tmem + kTmemS + 64u * (g & 1);
          uint32_t acc = 0;
#pragma unroll
          for (int box = 0; box < 4; ++box) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t ad = smem_desc_sw128(sQ + box * kQBoxBytes + ks * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(kvb + box * kKvBoxBytes + ks * 32, 16, 1024);
              umma_bf16_ss(dS, ad, bd, idesc_qk, acc);
              acc = 1;
            }
          }
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int ks = 2 * static_cast<int>(rank) + j;   // this CTA's 32 rope columns
            const uint64_t ad = smem_desc_sw128(sQ + 4 * kQBoxBytes + ks * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(kvb + 4 * kKvBoxBytes + ks * 32, 16, 1024);
            umma_bf16_ss(dS, ad, bd, idesc_qk, 1u);
          }
          mma_issued_any = true;
          umma_commit(&bars->sfull[g & 1]);
          if (i == hi - 1) umma_commit(&bars->qempty);
          if (pending >= 0 && !issue_pv(pending, pending_first)) { ok = false; break; }
          pending = g;
          pending_first = (i == lo);
        }
        ++segi;
      }
      if (ok && pending >= 0) issue_pv(pending, pending_first);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int q4 = warp & 3;                    // TMEM lane quarter this warp may access
    const int row = q4 * 32 + lane;             // row within the 128-row tile
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const uint32_t sX = smem_u32(smem + kOffX);
    const uint32_t sP = smem_u32(smem + kOffP);
    const uint32_t xrow = sX + row * 256;
    const uint32_t xrow_peer = mapa_shared(xrow, peer);
    const uint32_t peer_xfull = mapa_shared(smem_u32(&bars->xfull[q4]), peer);
    const uint32_t peer_xempty = mapa_shared(smem_u32(&bars->xempty[q4]), peer);
    const uint32_t prow = sP + (row >> 3) * 1024 + (row & 7) * 128;
    const float scale_log2 = p.scale_log2;
    const WsLayout wl = w;
    float* plse = reinterpret_cast<float*>(reinterpret_cast<char*>(p.ws) + wl.plse_off);
    float* po = reinterpret_cast<float*>(reinterpret_cast<char*>(p.ws) + wl.po_off);

    SegIter it{seq, p.batch, x0, x1, b_first};
    int g = 0, b, lo, hi;
    bool ok = true;
    while (ok && it.next(b, lo, hi)) {
      const int32_t* sq = seq + static_cast<size_t>(b) * kSeqWords;
      const int L = sq[kSeqLen];
      const int n_pages = sq[kSeqPages];
      const int rg = r_tile * kRowsPerTile + row;   // query row index (t, h)
      const int t = rg / p.heads;
      const int last_vis = L - p.q_len + t;         // query t sees tokens j <= L - T + t
      float m = -INFINITY, l = 0.f;
      for (int i = lo; i < hi; ++i, ++g) {
        if (!mbar_wait(&bars->sfull[g & 1], (g >> 1) & 1, tmo, abort_flag)) { ok = false; break; }
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

        // partial-S exchange with the peer CTA (row-swizzled to spread banks)
        if (g >= 1 && !mbar_wait<true>(&bars->xempty[q4], (g - 1) & 1, tmo, abort_flag)) { ok = false; break; }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint32_t ch = static_cast<uint32_t>(j ^ (row & 15));
          st_cluster_v4(xrow_peer + ch * 16, s[4 * j], s[4 * j + 1], s[4 * j + 2], s[4 * j + 3]);
        }
        mbar_arrive_remote(peer_xfull);
        if (!mbar_wait<true>(&bars->xfull[q4], g & 1, tmo, abort_flag)) { ok = false; break; }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint32_t ch = static_cast<uint32_t>(j ^ (row & 15));
          const float4 v = ld_shared_v4(xrow + ch * 16);
          s[4 * j] += v.x;
          s[4 * j + 1] += v.y;
          s[4 * j + 2] += v.z;
          s[4 * j + 3] += v.w;
        }
        mbar_arrive_remote(peer_xempty);

        // scale into the log2 domain; mask tokens past this query's position
        const int tok0 = i * kPage;
        if (tok0 + kPage - 1 > last_vis) {
#pragma unroll
          for (int j = 0; j < 64; ++j) s[j] = (tok0 + j <= last_vis) ? s[j] * scale_log2 : -INFINITY;
        } else {
#pragma unroll
          for (int j = 0; j < 64; ++j) s[j] *= scale_log2;
        }
        float mt = s[0];
#pragma unroll
        for (int j = 1; j < 64; ++j) mt = fmaxf(mt, s[j]);
        const float m_new = fmaxf(m, mt);
        float alpha = 1.f;
        bool resc = false;
        // Keep the running max unless it grows by more than 2^8: P stays <= 256.
        if (m_new > m + 8.f) {
          alpha = ex2_approx(m - m_new);
          resc = (i != lo);
          m = m_new;
        }
        const float mu = (m == -INFINITY) ? 0.f : m;
        float rs = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          s[j] = ex2_approx(s[j] - mu);
          rs += s[j];
        }
        l = l * alpha + rs;

        // PV(g-1) done: P buffer free and O stable.
        if (g >= 1 && !mbar_wait(&bars->pvdone, (g - 1) & 1, tmo, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
          const float a = resc ? alpha : 1.f;
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
        // Tail rows of the sequence's last page are not part of the context:
        // zero them in this CTA's V half so stale data (even NaN) cannot leak
        // through 0 * V in the PV product.
        if (i == n_pages - 1 && (L % kPage) != 0) {
          const int tail = L % kPage;
          uint8_t* vst = smem + kOffKV + (g % kStages) * kStageBytes;
          const int chunks = 4 * (kPage - tail) * 8;    // 16-byte chunks
          for (int idx = threadIdx.x - 64; idx < chunks; idx += 128) {
            const int box = idx / ((kPage - tail) * 8);
            const int rem = idx % ((kPage - tail) * 8);
            const int tok = tail + rem / 8;
            const int ch = rem % 8;
            st_shared_v4_u32(smem_u32(vst + box * kKvBoxBytes + tok * 128 + ch * 16), 0u, 0u, 0u, 0u);
          }
        }
        // P row -> bf16, 128B-swizzled K-major tile
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t ch = static_cast<uint32_t>(c ^ (row & 7));
          st_shared_v4_u32(prow + ch * 16, pack_bf16x2(s[8 * c], s[8 * c + 1]), pack_bf16x2(s[8 * c + 2], s[8 * c + 3]),
                           pack_bf16x2(s[8 * c + 4], s[8 * c + 5]), pack_bf16x2(s[8 * c + 6], s[8 * c + 7]));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->pfull);
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (!mbar_wait(&bars->pvdone, (g - 1) & 1, tmo, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const bool valid_row = rg < p.rows;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse_nat = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
      const int splits = sq[kSeqSplits];
      if (splits <= 1) {
        uint16_t* orow = p.out + (static_cast<size_t>(b) * p.rows + rg) * kDv + rank * 256;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_base + kTmemO + 32u * c, o);
          tc_wait_ld();
          if (valid_row) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pack_bf16x2(o[8 * v] * inv, o[8 * v + 1] * inv),
                                  pack_bf16x2(o[8 * v + 2] * inv, o[8 * v + 3] * inv),
                                  pack_bf16x2(o[8 * v + 4] * inv, o[8 * v + 5] * inv),
                                  pack_bf16x2(o[8 * v + 6] * inv, o[8 * v + 7] * inv));
          }
        }
        if (valid_row && rank == 0) p.lse[static_cast<size_t>(b) * p.rows + rg] = lse_nat;
      } else {
        const int slot = sq[kSeqSlot] + (c_idx - sq[kSeqFirstC]);
        const size_t pidx = (static_cast<size_t>(slot) * p.row_tiles + r_tile) * kRowsPerTile + row;
        float* orow = po + pidx * kDv + rank * 256;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_base + kTmemO + 32u * c, o);
          tc_wait_ld();
          float4* dst = reinterpret_cast<float4*>(orow + 32 * c);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(o[4 * v] * inv, o[4 * v + 1] * inv, o[4 * v + 2] * inv, o[4 * v + 3] * inv);
        }
        if (rank == 0) plse[pidx] = lse_nat;
      }
      tc_fence_before();
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncthreads();
  if (*abort_flag) {
    if (threadIdx.x == 0) atomicOr(&hdr[kHdrFlag], kFlagTimeout);
    // Let every copy and MMA this CTA started land before its memory goes away.
    if (warp == 0 && lane == 0) {
      for (int gg = max(0, tma_last_g - kStages + 1); gg <= tma_last_g; ++gg) {
        volatile int never = 0;
        mbar_wait(&bars->full[gg % kStages], (gg / kStages) & 1, kDrainTimeoutNs, &never);
      }
      if (tma_q_issued > 0) {
        volatile int never = 0;
        mbar_wait(&bars->qfull, (tma_q_issued - 1) & 1, kDrainTimeoutNs, &never);
      }
    }
    if (warp == 1 && lane == 0 && mma_issued_any) {
      umma_commit(&bars->drain);
      volatile int never = 0;
      mbar_wait(&bars->drain, 0, kDrainTimeoutNs, &never);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync_all();  // no CTA leaves while its peer may still touch its shared memory
}

}  // namespace

cudaError_t launch_decode_bf16(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const DecodeParams& p,
                               cudaStream_t stream) {
  // The dynamic shared-memory limit was raised for this device by
  // decode_bf16_max_active_clusters(), which the host API calls first.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.row_tiles * p.c_max, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mla_decode_bf16_kernel, tm_q, tm_kv, p);
}

cudaError_t decode_bf16_max_active_clusters(int* clusters) {
  cudaError_t e = cudaFuncSetAttribute(mla_decode_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(mla_decode_bf16_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
  (void)e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 1024, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(clusters, mla_decode_bf16_kernel, &cfg);
}

}  // namespace mla
