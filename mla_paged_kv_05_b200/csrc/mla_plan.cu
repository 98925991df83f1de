// K0: device-side split-KV planner.
//
// Reads the sequence lengths on the device (so a captured decode step needs
// no device-to-host round trip; zubnet.ai "LightSeek TokenSpeed 580 TPS ...
// B200", second paragraph: GPU-side sentinels instead of D2H syncs, whole
// decode loop in a CUDA graph) and cuts the concatenated page list of the
// batch into contiguous, equal-cost ranges, one per CTA-pair cluster, so that
// a single long context is spread over every SM.
//
// Cost model: sequence b costs n_b + kSeqOverhead units, its pages occupying
// positions [S_b + kSeqOverhead, S_b + kSeqOverhead + n_b) of a line of
// length total = sum_b cost_b. Cluster c owns positions [c*P, (c+1)*P) with
// P = max(kMinPayload, ceil(total / c_use)). A sequence whose pages fall in
// more than one cluster is "split": each piece writes an fp32 partial (O, lse)
// to its own slot and K2 merges them.
#include <cmath>
#include <mutex>

#include "mla_common.cuh"
#include "mla_launch.h"
#include "mla_ptx.cuh"

namespace mla {

namespace {

constexpr int kPlanThreads = 1024;

// Exclusive block-wide scan of one int per thread; returns the block total.
__device__ int block_exclusive_scan(int v, int* out_excl, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += n;
    }
    if (lane < nw) warp_tot[lane] = t;  // inclusive prefix of warp totals
  }
  __syncthreads();
  const int warp_excl = warp > 0 ? warp_tot[warp - 1] : 0;
  *out_excl = warp_excl + incl - v;
  const int total = warp_tot[(blockDim.x >> 5) - 1];
  __syncthreads();
  return total;
}

// The whole plan when the batch fits one thread per sequence: every per-sequence
// value stays in registers between the scans, and the clusters' first
// sequences are found by binary search over the cost prefix in shared memory.
// Same results as the general path below.
__device__ void plan_one_pass(const PlanParams& p, const WsLayout& w, int32_t* hdr, int32_t* first_b, int32_t* seq,
                              int* warp_tot) {
  __shared__ int ends[kPlanThreads];   // end of each sequence's cost interval
  const int b = threadIdx.x;
  const bool in = b < p.batch;
  int L = 0, n = 0, cost = 0;
  if (in) {
    L = p.seqlens[b];
    bool ok;
    plan_seq(L, p.q_len, p.max_pages, ok, n, cost);
    if (!ok) atomicOr(&hdr[kHdrFlag], kFlagBadSeqlen);
  }
  int start;
  const int total = block_exclusive_scan(cost, &start, warp_tot);
  const int payload = plan_payload(total, p.c_use);
  const int clusters = plan_clusters(total, payload);
  int splits = 0, first = 0;
  if (n > 0) plan_split(start, n, payload, first, splits);
  const bool listed = in && splits != 1;
  const int items = listed ? combine_items(splits, p.rows) : 0;
  int excl_slot, excl_list, excl_item;
  const int tot_slot = block_exclusive_scan(splits > 1 ? splits : 0, &excl_slot, warp_tot);
  const int tot_list = block_exclusive_scan(listed ? 1 : 0, &excl_list, warp_tot);
  const int tot_item = block_exclusive_scan(items, &excl_item, warp_tot);
  if (in) {
    int32_t* s = seq + static_cast<size_t>(b) * kSeqWords;
    s[kSeqStart] = start;
    s[kSeqPages] = n;
    s[kSeqLen] = L;
    s[kSeqFirstC] = first;
    s[kSeqSplits] = splits;
    s[kSeqSlot] = excl_slot;
    ends[b] = start + cost;
  }
  if (listed) {
    int32_t* list = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.list_off);
    int32_t* vcp = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.vcp_off);
    list[excl_list] = b;
    vcp[excl_list] = excl_item + items;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < p.c_max; c += blockDim.x) {
    int fb = p.batch;
    if (c < clusters) {
      const int x0 = c * payload;
      int lo = 0, hi = p.batch;   // smallest b with end_b > x0
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (ends[mid] > x0) hi = mid; else lo = mid + 1;
      }
      fb = lo;
    }
    first_b[c] = fb;
  }
  if (threadIdx.x == 0) {
    hdr[kHdrClusters] = clusters;
    hdr[kHdrPayload] = payload;
    hdr[kHdrTotal] = total;
    hdr[kHdrSlots] = tot_slot;
    hdr[kHdrListed] = tot_list;
    hdr[kHdrCombineCtas] = tot_item;
#ifdef MLA_TRACE
    if (p.trace != nullptr) p.trace[kTraceStepBase + 1] = static_cast<long long>(globaltimer_ns());
#endif
  }
}

// CTA k >= 1 of the planner grid: range-checks a strided share of the
// block-table entries the step will read (the first ceil(L_b / 64) of row b)
// against [0, num_pages). Its verdict goes to its own header word, rewritten
// every step (so nothing has to be cleared first); the decode kernel folds the
// words into the device flag.
__device__ void check_pages(const PlanParams& p, int32_t* hdr, int* warp_tot) {
  __shared__ int ends[kPlanThreads];   // per batch chunk: inclusive prefix of page counts
  const int k = blockIdx.x - 1;
  const int stride = p.check_ctas * static_cast<int>(blockDim.x);
  int bad = 0;
  for (int base = 0; base < p.batch; base += blockDim.x) {
    const int b = base + threadIdx.x;
    int n = 0;
    if (b < p.batch) {
      bool ok;
      int cost;
      plan_seq(p.seqlens[b], p.q_len, p.max_pages, ok, n, cost);
    }
    int excl;
    const int tot = block_exclusive_scan(n, &excl, warp_tot);
    ends[threadIdx.x] = excl + n;
    __syncthreads();
    const int nb = min(p.batch - base, static_cast<int>(blockDim.x));
    for (int u0 = k * static_cast<int>(blockDim.x) + threadIdx.x; u0 < tot; u0 += 4 * stride) {
      int id[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {   // four entries in flight per thread
        const int u = u0 + r * stride;
        id[r] = 0;
        if (u < tot) {
          int lo = 0, hi = nb - 1;   // the sequence whose page interval holds u
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (ends[mid] > u) hi = mid; else lo = mid + 1;
          }
          const int first = lo > 0 ? ends[lo - 1] : 0;
          id[r] = p.block_table[static_cast<size_t>(base + lo) * p.max_pages + (u - first)];
        }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) bad |= (id[r] < 0 || id[r] >= p.num_pages) ? 1 : 0;
    }
    __syncthreads();
  }
  bad = __syncthreads_or(bad);
  if (threadIdx.x == 0) hdr[kHdrCheck0 + k] = bad ? 1 : 0;
#ifdef MLA_TRACE
  if (threadIdx.x == 0 && p.trace != nullptr)
    atomicMax(reinterpret_cast<unsigned long long*>(p.trace) + kTraceStepBase + 5, globaltimer_ns());
#endif
}

// A checking warp of the one-warp planner (block k + 1 of its grid): the
// entries j = 32k + lane, stepping by 32 x check_ctas, of every sequence's
// first ceil(L_b / 64) block-table entries, four loads in flight per lane.
__device__ void check_pages_warp(const PlanParams& p, int32_t* hdr) {
  const int lane = threadIdx.x, k = blockIdx.x - 1;
  const int stride = 32 * p.check_ctas;
  int n = 0;
  if (lane < p.batch) {
    bool ok;
    int cost;
    plan_seq(p.seqlens[lane], p.q_len, p.max_pages, ok, n, cost);
  }
  int bad = 0;
  for (int b = 0; b < p.batch; ++b) {
    const int nb = __shfl_sync(0xffffffffu, n, b);
    const int32_t* row = p.block_table + static_cast<size_t>(b) * p.max_pages;
    for (int j0 = 32 * k + lane; j0 < nb; j0 += 4 * stride) {
      int id[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) id[r] = j0 + r * stride < nb ? row[j0 + r * stride] : 0;
#pragma unroll
      for (int r = 0; r < 4; ++r) bad |= (id[r] < 0 || id[r] >= p.num_pages) ? 1 : 0;
    }
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) hdr[kHdrCheck0 + k] = bad ? 1 : 0;
#ifdef MLA_TRACE
  if (lane == 0 && p.trace != nullptr)
    atomicMax(reinterpret_cast<unsigned long long*>(p.trace) + kTraceStepBase + 5, globaltimer_ns());
#endif
}

// The plan of a batch of at most 32 sequences by one warp (lane b = sequence
// b), with shuffles only: the CTA holds no shared memory, so it fits on an SM
// beside a 64-row decode CTA, which then does not wait for it (the decode
// kernel derives the same plan itself). Same results as plan_one_pass; blocks
// 1.. of the grid are checking warps.
__global__ void __launch_bounds__(32) mla_plan_warp_kernel(PlanParams p) {
  const WsLayout w = ws_layout(p.batch, p.row_tiles, p.c_max);
  int32_t* hdr = p.ws;
  int32_t* first_b = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.first_b_off);
  int32_t* seq = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.seq_off);
  const int lane = threadIdx.x;
#ifdef MLA_TRACE
  if (blockIdx.x == 0 && lane == 0 && p.trace != nullptr)
    p.trace[kTraceStepBase + 0] = static_cast<long long>(globaltimer_ns());
#endif
  pdl_launch_dependents();
  if (blockIdx.x > 0) {
    check_pages_warp(p, hdr);
    return;
  }
  if (lane == 0) {
    hdr[kHdrFlag] = 0;
    hdr[kHdrChecks] = p.check_ctas;
  }
  __syncwarp();
  const bool in = lane < p.batch;
  int L = 0, n = 0, cost = 0;
  if (in) {
    L = p.seqlens[lane];
    bool ok;
    plan_seq(L, p.q_len, p.max_pages, ok, n, cost);
    if (!ok) atomicOr(&hdr[kHdrFlag], kFlagBadSeqlen);
  }
  const int incl = warp_inclusive_scan(cost, lane);
  const int start = incl - cost;
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  const int payload = plan_payload(total, p.c_use);
  const int clusters = plan_clusters(total, payload);
  int splits = 0, first = 0;
  if (n > 0) plan_split(start, n, payload, first, splits);
  const bool listed = in && splits != 1;
  const int items = listed ? combine_items(splits, p.rows) : 0;
  const int sv = splits > 1 ? splits : 0;
  const int slot_incl = warp_inclusive_scan(sv, lane);
  const int item_incl = warp_inclusive_scan(items, lane);
  const unsigned lm = __ballot_sync(0xffffffffu, listed);
  const int excl_list = __popc(lm & ((1u << lane) - 1u));
  if (in) {
    int32_t* s = seq + static_cast<size_t>(lane) * kSeqWords;
    s[kSeqStart] = start;
    s[kSeqPages] = n;
    s[kSeqLen] = L;
    s[kSeqFirstC] = first;
    s[kSeqSplits] = splits;
    s[kSeqSlot] = slot_incl - sv;
  }
  if (listed) {
    int32_t* list = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.list_off);
    int32_t* vcp = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.vcp_off);
    list[excl_list] = lane;
    vcp[excl_list] = item_incl;
  }
  const int tot_slot = __shfl_sync(0xffffffffu, slot_incl, 31);
  const int tot_item = __shfl_sync(0xffffffffu, item_incl, 31);
  const int end = start + cost;   // the sequences' cost intervals end in batch order
  for (int c0 = 0; c0 < p.c_max; c0 += 32) {
    const int c = c0 + lane;
    const int x0 = c < clusters ? c * payload : 0;
    int fb = p.batch;   // first sequence whose interval ends after the cluster's start
    for (int b = 0; b < p.batch; ++b) {
      const int e = __shfl_sync(0xffffffffu, end, b);
      if (fb == p.batch && e > x0) fb = b;
    }
    if (c < p.c_max) first_b[c] = c < clusters ? fb : p.batch;
  }
  if (lane == 0) {
    hdr[kHdrClusters] = clusters;
    hdr[kHdrPayload] = payload;
    hdr[kHdrTotal] = total;
    hdr[kHdrSlots] = tot_slot;
    hdr[kHdrListed] = __popc(lm);
    hdr[kHdrCombineCtas] = tot_item;
#ifdef MLA_TRACE
    if (p.trace != nullptr) p.trace[kTraceStepBase + 1] = static_cast<long long>(globaltimer_ns());
#endif
  }
}

__global__ void __launch_bounds__(kPlanThreads) mla_plan_kernel(PlanParams p) {
  __shared__ int warp_tot[32];
  __shared__ int s_total, s_payload, s_clusters;
  const WsLayout w = ws_layout(p.batch, p.row_tiles, p.c_max);
  int32_t* hdr = p.ws;
  int32_t* first_b = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.first_b_off);
  int32_t* seq = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.seq_off);

#ifdef MLA_TRACE
  if (threadIdx.x == 0 && p.trace != nullptr) p.trace[kTraceStepBase + 0] = static_cast<long long>(globaltimer_ns());
#endif
  // The decode kernel may launch now; it waits for this grid's writes.
  pdl_launch_dependents();
  if (blockIdx.x > 0) {
    check_pages(p, hdr, warp_tot);
    return;
  }
  if (threadIdx.x == 0) {
    hdr[kHdrFlag] = 0;
    hdr[kHdrChecks] = p.check_ctas;
  }
  __syncthreads();
  if (p.batch <= static_cast<int>(blockDim.x)) {
    plan_one_pass(p, w, hdr, first_b, seq, warp_tot);
    return;
  }

  // Pass 1: page counts, validity, exclusive prefix of cost units.
  int carry = 0;
  for (int base = 0; base < p.batch; base += blockDim.x) {
    const int b = base + threadIdx.x;
    int L = 0, n = 0, cost = 0;
    if (b < p.batch) {
      L = p.seqlens[b];
      bool ok;
      plan_seq(L, p.q_len, p.max_pages, ok, n, cost);
      if (!ok) atomicOr(&hdr[kHdrFlag], kFlagBadSeqlen);
    }
    int excl;
    const int tot = block_exclusive_scan(cost, &excl, warp_tot);
    if (b < p.batch) {
      int32_t* s = seq + static_cast<size_t>(b) * kSeqWords;
      s[kSeqStart] = carry + excl;
      s[kSeqPages] = n;
      s[kSeqLen] = L;
    }
    carry += tot;
  }
  if (threadIdx.x == 0) {
    const int total = carry;
    const int payload = plan_payload(total, p.c_use);
    s_total = total;
    s_payload = payload;
    s_clusters = plan_clusters(total, payload);
  }
  __syncthreads();
  const int total = s_total, payload = s_payload, clusters = s_clusters;

  // Pass 2: clusters per sequence, partial-slot bases, and the combine list
  // (sequences with splits != 1: split ones, and invalid ones whose rows the
  // combine kernel fills with NaN) with its work-item prefix.
  int32_t* list = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.list_off);
  int32_t* vcp = reinterpret_cast<int32_t*>(reinterpret_cast<char*>(p.ws) + w.vcp_off);
  int slot_carry = 0, list_carry = 0, item_carry = 0;
  for (int base = 0; base < p.batch; base += blockDim.x) {
    const int b = base + threadIdx.x;
    int splits = 0, first = 0;
    if (b < p.batch) {
      const int32_t* s = seq + static_cast<size_t>(b) * kSeqWords;
      const int n = s[kSeqPages];
      if (n > 0) plan_split(s[kSeqStart], n, payload, first, splits);
    }
    const bool listed = b < p.batch && splits != 1;
    const int items = listed ? combine_items(splits, p.rows) : 0;
    int excl_slot, excl_list, excl_item;
    const int tot_slot = block_exclusive_scan(splits > 1 ? splits : 0, &excl_slot, warp_tot);
    const int tot_list = block_exclusive_scan(listed ? 1 : 0, &excl_list, warp_tot);
    const int tot_item = block_exclusive_scan(items, &excl_item, warp_tot);
    if (b < p.batch) {
      int32_t* s = seq + static_cast<size_t>(b) * kSeqWords;
      s[kSeqFirstC] = first;
      s[kSeqSplits] = splits;
      s[kSeqSlot] = slot_carry + excl_slot;
    }
    if (listed) {
      list[list_carry + excl_list] = b;
      vcp[list_carry + excl_list] = item_carry + excl_item + items;
    }
    slot_carry += tot_slot;
    list_carry += tot_list;
    item_carry += tot_item;
  }
  __syncthreads();

  // Pass 3: first sequence whose cost interval ends after each cluster's start.
  for (int c = threadIdx.x; c < p.c_max; c += blockDim.x) {
    int fb = p.batch;
    if (c < clusters) {
      const long long x0 = static_cast<long long>(c) * payload;
      int lo = 0, hi = p.batch;  // smallest b with end_b > x0
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        const int32_t* s = seq + static_cast<size_t>(mid) * kSeqWords;
        const int n = s[kSeqPages];
        const long long end = static_cast<long long>(s[kSeqStart]) + (n > 0 ? n + kSeqOverhead : 0);
        if (end > x0) hi = mid; else lo = mid + 1;
      }
      fb = lo;
    }
    first_b[c] = fb;
  }
  if (threadIdx.x == 0) {
    hdr[kHdrClusters] = clusters;
    hdr[kHdrPayload] = payload;
    hdr[kHdrTotal] = total;
    hdr[kHdrSlots] = slot_carry;
    hdr[kHdrListed] = list_carry;
    hdr[kHdrCombineCtas] = item_carry;
#ifdef MLA_TRACE
    if (p.trace != nullptr) p.trace[kTraceStepBase + 1] = static_cast<long long>(globaltimer_ns());
#endif
  }
}

}  // namespace

// The one-warp planner shares SMs with decode CTAs that hold ~223 KB of shared
// memory: it asks for the SM's whole unified memory as shared memory, so that
// an SM it lands on first is configured to take a decode CTA beside it.
cudaError_t warp_plan_attributes() {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (!done[dev]) {
    e = cudaFuncSetAttribute(mla_plan_warp_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

cudaError_t launch_plan(const PlanParams& p, cudaStream_t stream) {
  if (p.warp_plan) {
    const cudaError_t e = warp_plan_attributes();
    if (e != cudaSuccess) return e;
    mla_plan_warp_kernel<<<1 + p.check_ctas, 32, 0, stream>>>(p);
    return cudaGetLastError();
  }
  // One thread per sequence (whole warps) up to 1,024; the one-pass plan's
  // block-wide scans then cost no more than the batch needs.
  int threads = p.batch <= kPlanThreads ? ((p.batch < 1 ? 1 : p.batch) + 31) / 32 * 32 : kPlanThreads;
  if (p.check_ctas > 0 && threads < 512) threads = 512;   // the checking CTAs share the block size
  mla_plan_kernel<<<1 + p.check_ctas, threads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
