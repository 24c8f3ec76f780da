// fa_common.cuh -- pieces shared by the scheduler, forward and backward
// kernels and the host API: tile sizes, the workspace layout, sequence
// information from cumulative offsets, visible-tile ranges under the causal
// mask, and the bounded mbarrier wait.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/fa_varlen.h"
#include "sm100_ptx.cuh"

namespace fa {

// Forward tiles: a work item is 256 query rows of one (sequence, head),
// computed as two tiles of 128 rows that share every key tile; keys stream
// through in tiles of 128.
constexpr int kFwdBM = 128;
constexpr int kFwdBN = 128;
constexpr int kFwdItemRows = 256;
// Query rows per forward work item: head_dim 256 leaves TMEM room for one
// 128-row query tile per CTA only.
__host__ __device__ inline int fwd_item_rows(int D) { return D > 128 ? kFwdBM : kFwdItemRows; }
// Backward tiles: a work item is 128 key rows of one (sequence, head);
// queries stream through in tiles of 128.
constexpr int kBwdBN = 128;
constexpr int kBwdBM = 128;

// Per-call device state at the start of the workspace.
constexpr int kCostClasses = 12;  // cost classes [1, 2), [2, 4), ..., [2^11, inf)

struct WsHeader {
  uint32_t status;         // fa_status_t of the device side of the call
  uint32_t n_pairs;        // number of (sequence, tile) pairs in `pairs`
  uint32_t work_counter;   // next work item to hand out (reset by the scheduler)
  uint32_t work_counter2;  // the same, for a second kernel over the same list (head_dim 256 backward)
  // Cost-ordered lists: class_end[k] = number of pairs whose cost (visible
  // tiles on the other side) is at least 2^k; the pairs of cost class
  // [2^k, 2^(k+1)) are pairs[class_end[k+1] .. class_end[k]).
  uint32_t class_end[kCostClasses];
  uint32_t reserved[60 - kCostClasses];
};
static_assert(sizeof(WsHeader) == 256, "header is one 256-byte block");

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Upper bound on the number of (sequence, tile) pairs: sum_b ceil(len_b / T)
// <= total / T + batch.
__host__ __device__ inline int max_pairs(int batch, int total, int tile) { return total / tile + batch + 1; }

// Rows of the padded fp32 dQ accumulator per head: a query tile may run up
// to kBwdBM - 1 rows past the last token.
__host__ __device__ inline int dq_rows_padded(int total_q) { return static_cast<int>(align_up(total_q + kBwdBM, 64)); }

struct WsLayout {
  size_t seq_off;  // int32 [batch + 1]: first pair index of each sequence
  size_t pairs;    // int2  [max_pairs]: (sequence, tile), longest first
  size_t dvec;     // fp32  [H, tq_pad] (backward only): rowsum(dO * O)
  size_t qcount;   // u32   [H, tq_pad] (backward only): dQ additions done per query tile (deterministic mode)
  size_t dqacc;    // fp32  [H, tq_pad, D] (backward only)
  size_t total;
  int max_pairs;
  int tq_pad;
};

__host__ __device__ inline WsLayout ws_layout(bool backward, int batch, int total_q, int total_k, int H, int D) {
  WsLayout L{};
  size_t off = sizeof(WsHeader);
  L.seq_off = off;
  off = align_up(off + sizeof(int32_t) * (static_cast<size_t>(batch) + 1), 256);
  L.max_pairs = backward ? max_pairs(batch, total_k, kBwdBN) : max_pairs(batch, total_q, fwd_item_rows(D));
  L.pairs = off;
  off = align_up(off + 8 * static_cast<size_t>(L.max_pairs), 256);
  if (backward) {
    L.tq_pad = dq_rows_padded(total_q);
    L.dvec = off;
    off = align_up(off + sizeof(float) * static_cast<size_t>(H) * L.tq_pad, 256);
    L.qcount = off;
    off = align_up(off + sizeof(uint32_t) * static_cast<size_t>(H) * L.tq_pad, 256);
    L.dqacc = off;
    off = align_up(off + sizeof(float) * static_cast<size_t>(H) * L.tq_pad * D, 256);
  }
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- sequences
// Page "Mecanismo cu_seqlens en FlashAttention", "Lógica de cálculo de
// longitud": query sequence b starts at packed row cu_q[b] and has
// cu_q[b+1] - cu_q[b] rows. Its keys are found one of two ways:
//  * packed (cumulative offsets): rows cu_k[b] .. cu_k[b+1]-1 of the key
//    tensor;
//  * key/value cache (per-sequence lengths, not cumulative, with left
//    padding): sequence b owns a slot of cache_rows rows starting at row
//    b*cache_rows, and its keys are slot rows leftpad_k[b] .. seqlens_k[b]-1,
//    so it has seqlens_k[b] - leftpad_k[b] of them;
//  * paged key/value cache (the pages' "caché KV paginada"): seqlens_k[b]
//    keys whose position p lives in page block_table[b][p / page_size] at
//    row p % page_size; the pool is pages of page_size rows, back to back.
struct KeyRows {
  const int32_t* cu_k;         // packed layout: [batch + 1] cumulative offsets
  const int32_t* seqlens_k;    // cache layouts: [batch] key counts (incl. padding) (null: packed)
  const int32_t* leftpad_k;    // cache layout: [batch] left padding, or null (none)
  int cache_rows;              // cache layout: rows per sequence slot
  const int32_t* block_table;  // paged layout: [batch, max_pages] page indices (null: not paged)
  int max_pages;               // paged layout: block-table entries per sequence
  int page_size;               // paged layout: rows per page (a multiple of kFwdBN)
};

struct SeqInfo {
  int q0, lq, k0, lk;
};

// The three key layouts, for kernels specialised on one of them.
enum KeyLayout : int { kKeysPacked = 0, kKeysSlots = 1, kKeysPaged = 2 };
__host__ __device__ inline int key_layout(const KeyRows& kr) {
  return kr.block_table ? kKeysPaged : (kr.seqlens_k ? kKeysSlots : kKeysPacked);
}
template <int KL>
__device__ __forceinline__ SeqInfo seq_info_l(const int32_t* cu_q, const KeyRows& kr, int b) {
  SeqInfo s;
  s.q0 = __ldg(cu_q + b);
  s.lq = __ldg(cu_q + b + 1) - s.q0;
  if (KL == kKeysPaged) {
    s.k0 = 0;  // rows come from the block table (key_tile_row)
    s.lk = __ldg(kr.seqlens_k + b);
  } else if (KL == kKeysSlots) {
    const int lp = kr.leftpad_k ? __ldg(kr.leftpad_k + b) : 0;
    s.k0 = b * kr.cache_rows + lp;
    s.lk = __ldg(kr.seqlens_k + b) - lp;
  } else {
    s.k0 = __ldg(kr.cu_k + b);
    s.lk = __ldg(kr.cu_k + b + 1) - s.k0;
  }
  return s;
}

__device__ __forceinline__ SeqInfo seq_info(const int32_t* cu_q, const KeyRows& kr, int b) {
  SeqInfo s;
  s.q0 = __ldg(cu_q + b);
  s.lq = __ldg(cu_q + b + 1) - s.q0;
  if (kr.block_table) {
    s.k0 = 0;  // rows come from the block table (key_tile_row)
    s.lk = __ldg(kr.seqlens_k + b);
  } else if (kr.seqlens_k) {
    const int lp = kr.leftpad_k ? __ldg(kr.leftpad_k + b) : 0;
    s.k0 = b * kr.cache_rows + lp;
    s.lk = __ldg(kr.seqlens_k + b) - lp;
  } else {
    s.k0 = __ldg(kr.cu_k + b);
    s.lk = __ldg(kr.cu_k + b + 1) - s.k0;
  }
  return s;
}

// Row, in the key/value tensor, of the first key of key tile j (tiles of bn
// keys) of sequence b. A tile never straddles two pages: the page size is a
// multiple of 128, hence of bn.
__device__ __forceinline__ int key_tile_row(const KeyRows& kr, int b, const SeqInfo& s, int j, int bn = kFwdBN) {
  if (kr.block_table) {
    const int pos = j * bn;
    const int page = __ldg(kr.block_table + static_cast<size_t>(b) * kr.max_pages + pos / kr.page_size);
    return page * kr.page_size + pos % kr.page_size;
  }
  return s.k0 + j * bn;
}

// Number of key tiles (kFwdBN keys) visible from the query rows below
// row_end (clamped to lq), given the bottom-right causal rule
// j <= i + (lk - lq). Tiles wholly above the diagonal are skipped; the
// visible tiles are always a prefix 0 .. n-1.
__host__ __device__ inline int fwd_k_tiles(int row_end, int lq, int lk, bool causal, int bn = kFwdBN) {
  if (lk <= 0 || lq <= 0) return 0;
  const int nk = (lk + bn - 1) / bn;
  if (!causal) return nk;
  const int rmax = (row_end < lq ? row_end : lq) - 1;
  const long long last = static_cast<long long>(rmax) + lk - lq;
  if (last < 0) return 0;
  const long long n = last / bn + 1;
  return n < nk ? static_cast<int>(n) : nk;
}

// Range [begin, end) of backward query tiles (bm rows) that see at least
// one key of key tile j (keys j*BN ..).
__host__ __device__ inline void bwd_q_tiles(int j, int lq, int lk, bool causal, int* begin, int* end,
                                            int bm = kBwdBM) {
  const int nq = (lq + bm - 1) / bm;
  *end = nq;
  *begin = 0;
  if (lk <= 0 || lq <= 0) {
    *begin = nq;
    return;
  }
  if (causal) {
    long long first = static_cast<long long>(j) * kBwdBN - (lk - lq);
    if (first < 0) first = 0;
    *begin = first >= lq ? nq : static_cast<int>(first / bm);
  }
}

// --------------------------------------------------------- bounded waits
// Every pipeline wait gives up after a time limit (a kernel argument, this
// long unless a test shortens it), records FA_ERR_DEVICE_TIMEOUT in the
// workspace status and raises the CTA's abort flag so the other roles stop
// too.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;

struct Abort {
  volatile int* flag;  // shared memory, one per CTA
  uint32_t* status;    // workspace status word
  uint64_t limit_ns;   // time limit of every wait
};

__device__ __forceinline__ void raise_abort(const Abort& ab) {
  *ab.flag = 1;
  atomicCAS(ab.status, 0u, static_cast<uint32_t>(FA_ERR_DEVICE_TIMEOUT));
}

static __device__ __forceinline__ bool wait_slow(uint32_t addr, uint32_t parity, const Abort& ab) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(addr, parity)) return true;
    if (*ab.flag) return false;
    if (globaltimer_ns() - t0 > ab.limit_ns) {
      raise_abort(ab);
      return false;
    }
  }
}

// Wait for the phase of `bar` with the given parity to complete. Returns
// false if the CTA is aborting (the caller must stop its role).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Abort& ab) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try_wait(addr, parity)) return true;
  return wait_slow(addr, parity, ab);
}

// Exit-path wait for work this thread itself put in flight (TMA loads,
// MMAs): ignores the abort flag and gives up only after the time limit.
__device__ __forceinline__ static bool wait_bar_final(uint64_t* bar, uint32_t parity, const Abort& ab) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(addr, parity)) return true;
    if (globaltimer_ns() - t0 > ab.limit_ns) {
      raise_abort(ab);
      return false;
    }
  }
}

// Warp-uniform form for roles whose next step is a .sync.aligned tcgen05
// instruction: every lane returns the same answer.
__device__ __forceinline__ bool wait_bar_warp(uint64_t* bar, uint32_t parity, const Abort& ab) {
  const bool ok = wait_bar(bar, parity, ab);
  return __all_sync(0xffffffffu, ok);
}

// ------------------------------------------------------- dynamic work items
// Persistent CTAs take work items (in the scheduler's longest-first order)
// from a global counter. One thread per CTA claims each item and publishes
// its index to the CTA's other roles through this ring; -1 means "no more".
constexpr int kItemSlots = 4;
struct ItemRing {
  uint64_t full[kItemSlots];   // count 1: the publishing thread
  uint64_t empty[kItemSlots];  // count = number of consuming arrivals per item
  int idx[kItemSlots];
};

__device__ __forceinline__ void item_ring_init(ItemRing& r, uint32_t consumers) {
  for (int i = 0; i < kItemSlots; ++i) {
    mbar_init(&r.full[i], 1);
    mbar_init(&r.empty[i], consumers);
  }
}

// Publisher (one thread): claim the next item and publish it. Returns false
// if the CTA is aborting.
__device__ __forceinline__ bool publish_item(ItemRing& r, uint32_t& n, uint32_t* counter, int n_items, int& idx,
                                             const Abort& ab) {
  const int slot = n % kItemSlots;
  if (n >= kItemSlots && !wait_bar(&r.empty[slot], ((n / kItemSlots) - 1) & 1, ab)) return false;
  int v = static_cast<int>(atomicAdd(counter, 1u));
  if (v >= n_items) v = -1;
  *reinterpret_cast<volatile int*>(&r.idx[slot]) = v;
  mbar_arrive(&r.full[slot]);
  ++n;
  idx = v;
  return true;
}

// Publisher that also decodes each claimed item once for all roles: for a
// claimed index, `decode(slot, idx)` stores the decoded item beside the ring
// before it is published (the mbarrier arrive orders those writes before the
// consumers' wait), and consumers copy it out before releasing the slot.
template <typename Decode>
__device__ __forceinline__ bool publish_item_decoded(ItemRing& r, uint32_t& n, uint32_t* counter, int n_items,
                                                     int& idx, const Abort& ab, Decode&& decode) {
  const int slot = n % kItemSlots;
  if (n >= kItemSlots && !wait_bar(&r.empty[slot], ((n / kItemSlots) - 1) & 1, ab)) return false;
  int v = static_cast<int>(atomicAdd(counter, 1u));
  if (v >= n_items) v = -1;
  if (v >= 0) decode(slot, v);
  *reinterpret_cast<volatile int*>(&r.idx[slot]) = v;
  mbar_arrive(&r.full[slot]);
  ++n;
  idx = v;
  return true;
}

// Consumer: wait for the n-th published item; returns its index, or -1 when
// there is no more work (or the CTA is aborting). `slot` receives the ring
// slot, on whose `empty` barrier the caller arrives once it has the index.
template <bool WARP>
__device__ __forceinline__ int consume_item(ItemRing& r, uint32_t& n, int& slot, const Abort& ab) {
  slot = n % kItemSlots;
  const uint32_t par = (n / kItemSlots) & 1;
  const bool ok = WARP ? wait_bar_warp(&r.full[slot], par, ab) : wait_bar(&r.full[slot], par, ab);
  ++n;
  if (!ok) return -2;
  return *reinterpret_cast<volatile int*>(&r.idx[slot]);
}

// kern<<<grid, block, smem, stream>>>(args...). With `chained` the grid is a
// programmatic dependent of the kernel before it in the stream: it may be
// scheduled (and run its prologue: barriers, tensor memory, descriptor
// prefetch) while that kernel still runs, and every one of its threads
// executes griddep_wait() before it reads or writes memory that kernel (or
// anything before it) touches.
template <class... KArgs, class... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), unsigned grid, unsigned block, size_t smem,
                                 cudaStream_t stream, bool chained, const Args&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr = {};
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = chained ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

}  // namespace fa
