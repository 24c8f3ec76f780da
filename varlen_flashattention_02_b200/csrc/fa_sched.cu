// fa_sched.cu -- work-list preparation for the persistent attention kernels.
//
// From the device-resident cumulative offsets, one CTA
//   1. checks them (cu[0] = 0, non-decreasing, cu[batch] = total, every
//      length <= max_seqlen; for a key/value cache 0 <= leftpad_k[b] <=
//      seqlens_k[b] <= cache_rows; for a paged cache every page a sequence
//      uses inside the pool) and records FA_ERR_BAD_SEQLENS otherwise;
//   2. counts the tiles of every sequence (forward: query blocks of 256
//      rows; backward: key tiles of 128 rows) and prefix-sums them;
//   3. orders all (sequence, tile) pairs by their number of visible tiles on
//      the other side, most work first, so that the persistent kernels,
//      which take pairs in order, start the longest items first (or, for
//      the deterministic backward, keeps (sequence, tile) order).
// No padding is ever enumerated: a sequence of length n yields ceil(n/T)
// pairs (T = 256 forward, 128 backward). Pages: "Mecanismo cu_seqlens en
// FlashAttention", "Lógica de cálculo de longitud" (lengths from offsets)
// and "Consejos de optimización" (long and short sequences mixed in one
// batch); "Flash-Atención y Flash-Atención-2", FlashAttention-2 section
// (parallelism over the sequence dimension as well as batch and heads).
#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {
namespace {

constexpr int kThreads = 1024;
constexpr int kBins = 2048;  // cost buckets; costs above kBins-1 share the last

__device__ __forceinline__ int pair_cost(const SeqInfo& s, int tile, int mode, int rows, bool causal) {
  if (mode == 0) return fwd_k_tiles((tile + 1) * rows, s.lq, s.lk, causal);
  int b, e;
  bwd_q_tiles(tile, s.lq, s.lk, causal, &b, &e);
  return e - b;
}

// Block-wide inclusive scan of one int per thread.
__device__ __forceinline__ int block_inclusive_scan(int v, int* s_warp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = s_warp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    s_warp[lane] = w;
  }
  __syncthreads();
  const int r = v + (warp > 0 ? s_warp[warp - 1] : 0);
  __syncthreads();
  return r;
}

// Largest b with seq_off[b] <= p (seq_off non-decreasing, seq_off[batch] > p).
__device__ __forceinline__ int find_seq(const int32_t* seq_off, int batch, int p) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seq_off[mid] <= p)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kThreads) sched_prep_kernel(SchedArgs a) {
  __shared__ int s_hist[kBins];
  __shared__ int s_warp[32];
  __shared__ int s_err;
  __shared__ int s_total;
  __shared__ int s_max_tiles;
  auto* hdr = reinterpret_cast<WsHeader*>(a.workspace);
  auto* seq_off = reinterpret_cast<int32_t*>(static_cast<char*>(a.workspace) + a.seq_off_offset);
  auto* pairs = reinterpret_cast<int2*>(static_cast<char*>(a.workspace) + a.pairs_offset);
  const int tid = threadIdx.x;
  const bool causal = a.causal != 0;
  // The attention kernel launched behind this one may take its SMs and run
  // its prologue now; it waits for this grid before it reads the work list.
  griddep_launch_dependents();

  const bool cache = a.keys.seqlens_k != nullptr;
  if (tid == 0) {
    s_err = 0;
    s_total = 0;
    s_max_tiles = 0;
    hdr->work_counter = 0;
    hdr->work_counter2 = 0;
    if (a.cu_q[0] != 0 || a.cu_q[a.batch] != a.total_q) s_err = 1;
    if (!cache && (a.keys.cu_k[0] != 0 || a.keys.cu_k[a.batch] != a.total_k)) s_err = 1;
  }
  for (int i = tid; i < kBins; i += kThreads) s_hist[i] = 0;
  __syncthreads();
  for (int b = tid; b < a.batch; b += kThreads) {
    const int lq = a.cu_q[b + 1] - a.cu_q[b];
    int lk;
    if (a.keys.block_table) {
      // 0 <= seqlens_k <= max_pages * page_size, and every page it uses
      // inside the pool.
      lk = a.keys.seqlens_k[b];
      if (lk < 0 || lk > a.keys.max_pages * a.keys.page_size) {
        s_err = 1;
      } else {
        const int n_pages = (lk + a.keys.page_size - 1) / a.keys.page_size;
        const int pool_pages = a.total_k / a.keys.page_size;
        for (int i = 0; i < n_pages; ++i) {
          const int pg = a.keys.block_table[static_cast<size_t>(b) * a.keys.max_pages + i];
          if (pg < 0 || pg >= pool_pages) s_err = 1;
        }
      }
    } else if (cache) {
      // 0 <= leftpad <= seqlens_k <= cache_rows.
      const int lp = a.keys.leftpad_k ? a.keys.leftpad_k[b] : 0;
      const int sl = a.keys.seqlens_k[b];
      if (lp < 0 || sl < lp || sl > a.keys.cache_rows) s_err = 1;
      lk = sl - lp;
    } else {
      lk = a.keys.cu_k[b + 1] - a.keys.cu_k[b];
    }
    if (lq < 0 || lk < 0 || lq > a.max_seqlen_q || lk > a.max_seqlen_k) s_err = 1;
  }
  __syncthreads();
  if (s_err) {
    if (tid == 0) {
      hdr->status = FA_ERR_BAD_SEQLENS;
      hdr->n_pairs = 0;
    }
    return;
  }

  // Tiles per sequence, exclusive prefix sum into seq_off.
  const int tile = a.mode == 0 ? a.item_rows : kBwdBN;
  for (int base = 0; base < a.batch; base += kThreads) {
    const int b = base + tid;
    int n = 0;
    if (b < a.batch) {
      const int len = a.mode == 0 ? a.cu_q[b + 1] - a.cu_q[b] : a.keys.cu_k[b + 1] - a.keys.cu_k[b];
      n = (len + tile - 1) / tile;
      atomicMax(&s_max_tiles, n);
    }
    const int incl = block_inclusive_scan(n, s_warp);
    if (b < a.batch) seq_off[b] = s_total + incl - n;
    __syncthreads();
    if (tid == kThreads - 1) s_total += incl;
    __syncthreads();
  }
  const int n_pairs = s_total;
  if (tid == 0) seq_off[a.batch] = n_pairs;
  if (n_pairs > a.max_pairs) {  // cannot happen for valid offsets; defensive
    if (tid == 0) {
      hdr->status = FA_ERR_BAD_SEQLENS;
      hdr->n_pairs = 0;
    }
    return;
  }
  __syncthreads();

  // Tile-major order (deterministic backward): every sequence's tile 0, then
  // every tile 1, ...; the tiles of one sequence are then claimed in
  // increasing order, which is what the deterministic dQ turn-taking needs
  // (the order among sequences does not matter to the result). Tile 0 sees
  // the most queries under the causal mask, so this is also longest first.
  // Sequences with more tiles than histogram buckets fall back to plain
  // (sequence, tile) order.
  const bool tile_major = a.natural_order && s_max_tiles <= kBins;
  if (a.natural_order && !tile_major) {
    for (int p = tid; p < n_pairs; p += kThreads) {
      const int b = find_seq(seq_off, a.batch, p);
      pairs[p] = make_int2(b, p - seq_off[b]);
    }
    if (tid == 0) {
      hdr->status = FA_OK;
      hdr->n_pairs = static_cast<uint32_t>(n_pairs);
    }
    return;
  }

  // Histogram of costs.
  for (int p = tid; p < n_pairs; p += kThreads) {
    const int b = find_seq(seq_off, a.batch, p);
    const SeqInfo s = seq_info(a.cu_q, a.keys, b);
    const int t = p - seq_off[b];
    const int c = tile_major ? kBins - 1 - t : min(pair_cost(s, t, a.mode, a.item_rows, causal), kBins - 1);
    atomicAdd(&s_hist[c], 1);
  }
  __syncthreads();

  // Start offset of every bucket, highest cost first.
  {
    constexpr int per = kBins / kThreads;
    int v[per];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) {
      v[i] = s_hist[kBins - 1 - (tid * per + i)];
      sum += v[i];
    }
    const int incl = block_inclusive_scan(sum, s_warp);
    int run = incl - sum;
#pragma unroll
    for (int i = 0; i < per; ++i) {
      s_hist[kBins - 1 - (tid * per + i)] = run;
      run += v[i];
    }
  }
  __syncthreads();

  // Cost classes: s_hist[c] now counts the pairs of cost above c.
  static_assert(kBins == 1 << (kCostClasses - 1), "the top class starts at the last bucket");
  const int class_end = tid < kCostClasses ? s_hist[(1 << tid) - 1] : 0;
  __syncthreads();

  // Scatter.
  for (int p = tid; p < n_pairs; p += kThreads) {
    const int b = find_seq(seq_off, a.batch, p);
    const SeqInfo s = seq_info(a.cu_q, a.keys, b);
    const int t = p - seq_off[b];
    const int c = tile_major ? kBins - 1 - t : min(pair_cost(s, t, a.mode, a.item_rows, causal), kBins - 1);
    const int pos = atomicAdd(&s_hist[c], 1);
    pairs[pos] = make_int2(b, t);
  }
  if (tid < kCostClasses) hdr->class_end[tid] = tile_major ? 0u : static_cast<uint32_t>(class_end);
  if (tid == 0) {
    hdr->status = FA_OK;
    hdr->n_pairs = static_cast<uint32_t>(n_pairs);
  }
}

}  // namespace

cudaError_t launch_sched_prep(const SchedArgs& a, cudaStream_t stream) {
  sched_prep_kernel<<<1, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fa
