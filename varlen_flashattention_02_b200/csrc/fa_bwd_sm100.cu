// fa_bwd_sm100.cu -- backward varlen attention for sm_100a (head_dim 64, 128).
//
// Three kernels per call, after the work-list preparation (key-tile mode):
//  1. preprocess: Dv_i = sum_c dO_ic * O_ic (fp32, [H, rows]) and zero the
//     fp32 dQ accumulator;
//  2. main: one persistent CTA per SM takes (sequence, key/value head,
//     key-tile) items, longest first, from a global counter. For 128 keys
//     K_j, V_j of one key/value head it loops over the query heads that read
//     that head (one, or a group under grouped-query attention) and the
//     128-row query tiles that see the keys, recomputing the probabilities
//     from the saved logsumexp instead of storing them:
//        S^T  = K_j Q_i^T,  P^T = exp2(S^T*scale*log2e - lse_i*log2e)
//        dP^T = V_j dO_i^T, dS^T = P^T * (dP^T - Dv_i)
//        dV_j += P^T dO_i,  dK_j += dS^T Q_i      (accumulated in TMEM)
//        dQ_i^T = K_j^T dS^T -> added to the fp32 accumulator in global
//                               memory with bulk reductions
//     and finally writes dK_j = scale * dK_j and dV_j as bf16;
//  3. convert: dQ = bf16(scale * dQacc).
//
// Pages: "Flash-Atención y Flash-Atención-2", FlashAttention v1 section
// (tiling and recomputation: probabilities are recomputed in the backward)
// and backward paragraph (each worker owns a block of columns of the
// attention matrix, i.e. a key tile; workers aggregate the query gradient
// with atomic operations, which beats row parallelism that would have to
// aggregate dK and dV); "Mecanismo cu_seqlens en FlashAttention" (per-
// sequence offsets and lengths from the cumulative arrays). The gradient
// formulas are the chain rule of softmax attention (the pages print none).
//
// B200 design. Each step works on 128 keys x 128 queries, so every MMA is
// M = 128 with N = 128 (or N = head_dim): five groups of D/16 or 8 MMAs per
// step. Warp roles (16 warps): warp 0 TMA loads and item claims, warp 1 MMA
// issue, warps 2-3 stage logsumexp/Dv rows, two P/dS warpgroups (warps 4-7:
// queries 0-63 of the step, warps 8-11: queries 64-127; one thread per key
// row = TMEM lane), warps 12-15 drain dQ^T into bulk fp32 reductions and
// write dK/dV. Tensor memory holds dK, dV, S^T and dP^T; P^T and dS^T are
// written back over their S^T columns as bf16 so that both the dV and the dK
// MMA read their A operand from TMEM; dS^T also goes to shared memory once,
// as the B operand of dQ^T = K^T dS^T, whose result reuses the dP^T columns.
// Once a step's MMAs have completed, its Q/dO stage (exactly the size of the
// step's fp32 dQ tile) is the staging area of that step's dQ reduction, and
// at an item's end of its dK/dV stores; the drain group then hands the stage
// back to the loader. At head_dim 128 shared memory holds K, V, two Q/dO
// stages and the dS^T tile: the whole 227 KB.
#include <type_traits>

#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {
namespace {

constexpr int BN = kBwdBN;  // keys per item
constexpr int BM = kBwdBM;  // queries per step
static_assert(BN == 128 && BM == 128, "one 128 x 128 tile per step");
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
// TMEM column map: dK, dV (D columns each), S^T (P^T at +0/+64, dS^T at
// +32/+96 as bf16 pairs, one 64-query half per P/dS warpgroup), dP^T (then
// dQ^T: D lanes x 128 query columns).
constexpr int kColDP = 384;  // dP^T of the step, then its dQ^T
// TMEM columns of the dK and dV accumulators and of the S^T buffer(s). At
// head_dim 64 the accumulators take 64 columns each and a second S^T buffer
// fits: step p uses buffer p & 1, and the next step's S^T is computed while
// this step's dS^T is being formed, so the P/dS warps go from dS^T of one
// step straight to P^T of the next.
template <int D>
struct TCols {
  static constexpr bool kTwoS = D == 64;
  static constexpr uint32_t dk = 0, dv = D == 64 ? 64 : 128;
  static constexpr uint32_t s0 = D == 64 ? 128 : 256;
  __device__ static constexpr uint32_t s(uint32_t p) { return kTwoS ? s0 + (p & 1u) * 128u : s0; }
  // s_full barrier of step p and the parity of its wait.
  __device__ static constexpr int sbar(uint32_t p) { return kTwoS ? static_cast<int>(p & 1u) : 0; }
  __device__ static constexpr uint32_t spar(uint32_t p) { return kTwoS ? (p >> 1) & 1u : p & 1u; }
};
static_assert(TCols<64>::s0 + 256 <= kColDP && TCols<128>::s0 + 128 <= kColDP, "TMEM columns");
constexpr int kPdsWarp0 = 4, kDrainWarp0 = 12;

template <int D>
struct BwdSmem {
  static constexpr int kQStages = D == 64 ? 3 : 2;  // Q/dO stages (and logsumexp/Dv slots) in flight
  static constexpr int kChunks = D / 64;
  static constexpr int kKChunk = BN * 128;  // [128 rows x 64 bf16] swizzled chunk
  static constexpr int kQChunk = BM * 128;
  static constexpr int kKTile = kChunks * kKChunk;
  static constexpr int kQTile = kChunks * kQChunk;
  static constexpr int kDsHalf = BN * 64 * 2;  // dS^T [128 keys x 64 queries] bf16, one swizzled chunk
  static constexpr int kDsTile = 2 * kDsHalf;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kKTile;
  static constexpr int kQdo = kV + kKTile;  // stage s: Q at kQdo + 2s*QTile, dO after it
  static constexpr int kDs = kQdo + 2 * kQStages * kQTile;
  static constexpr int kLd = kDs + kDsTile;  // slots x (lse[128], dv[128]) fp32
  static constexpr int kBar = kLd + kQStages * 2 * BM * 4;
  static constexpr int kBytes = kBar + 512;
};
static_assert(BwdSmem<128>::kBytes <= 232448 && BwdSmem<64>::kBytes <= 232448, "layout fits 227 KB");
// A Q/dO stage holds a step's fp32 dQ tile (128 queries x D) and a key
// tile's bf16 dV and dK (2 x 128 x D).
static_assert(2 * BwdSmem<128>::kQTile == BM * 128 * 4 && 2 * BwdSmem<64>::kQTile == BM * 64 * 4, "stage");

// An item is (sequence, key/value head hk, key tile j). Its steps visit the
// query tiles i0 .. i0+nt-1 that see the key tile, for each query head of
// hk's group in turn: step s is query head h0 + s / nt, tile i0 + s % nt.
// dK and dV of the tile accumulate over all of them.
struct Item {
  int b, hk, j;
  SeqInfo s;
  int i0, nt;  // first query tile and query tiles per head
  int h0;      // first query head of the group
  int n;       // steps: nt * group
};

// Work order. The items are the work list's (sequence, key tile) pairs,
// most query tiles first, each for every key/value head, claimed in index
// order. Plain order: item idx is pair idx / Hk of head idx % Hk, so the
// longest items of all heads start first. Class order (CLASSES): the pairs
// fall into cost classes [2^k, 2^(k+1)) (class_end from the work-list
// kernel); the classes are taken longest first, and within a class head by
// head. Concurrent items then mostly share a head, whose Q/dO tiles and part
// of the fp32 dQ accumulator stay in L2 while they are read and reduced
// into, while no item can start much later than one twice as long.
template <bool CLASSES>
__device__ __forceinline__ Item get_item(const BwdArgs& a, const int2* pairs, int idx, int n_pairs,
                                         const uint32_t* class_end) {
  Item it;
  int pair = idx / a.Hk, hk = idx % a.Hk;
  if constexpr (CLASSES) {
    int lo = 0;  // pairs of the classes before this one
#pragma unroll
    for (int k = kCostClasses - 1; k >= -1; --k) {
      const int hi = k >= 0 ? static_cast<int>(class_end[k]) : n_pairs;
      if (idx < hi * a.Hk) {
        const int n = hi - lo, local = idx - lo * a.Hk;
        hk = local / n;
        pair = lo + local % n;
        break;
      }
      lo = hi;
    }
  }
  const int2 pr = pairs[pair];
  it.hk = hk;
  it.h0 = it.hk * a.group;
  it.b = pr.x;
  it.j = pr.y;
  it.s = seq_info(a.cu_q, a.keys, it.b);
  int e;
  bwd_q_tiles(it.j, it.s.lq, it.s.lk, a.causal != 0, &it.i0, &e);
  it.nt = e - it.i0;
  it.n = it.nt * a.group;
  return it;
}

struct Bars {
  uint64_t kv_full, kv_empty;
  // Q and dO halves of each stage, filled and released separately: the
  // drain hands the Q half back as soon as the first half of the step's dQ
  // reduction has read it, so the next Q load starts early.
  uint64_t q_full[3], q_empty[3], do_full[3], do_empty[3];
  uint64_t s_full[2], dp_full;  // S^T (per buffer), dP^T of the step in TMEM
  uint64_t p_full, ds_full;   // P^T (TMEM), dS^T (TMEM and shared) written
  uint64_t dq_full, dq_free;  // dQ^T in TMEM; read out by the drain group
  uint64_t dkv_full, dv_free, dk_free;
  uint64_t ld_full[3], ld_empty[3];
  uint64_t drain;
  ItemRing items;
  Item item_data[kItemSlots];  // the published items, decoded once by the producer
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block fits its reserved space");

// Query head and query tile of step s of an item.
struct Step {
  int h, t;
};
__device__ __forceinline__ Step item_step(const Item& it, int s) {
  const int r = s / it.nt;
  return Step{it.h0 + r, it.i0 + s - r * it.nt};
}

// Deterministic mode: wait until the dQ additions of key tiles 0 .. j-1 to
// the query tile whose counter is `cnt` are done (bounded, like every wait).
__device__ __forceinline__ bool wait_dq_turn(const uint32_t* cnt, uint32_t j, const Abort& ab) {
  if (ld_acquire_gpu(cnt) >= j) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (ld_acquire_gpu(cnt) >= j) return true;
    if (*ab.flag) return false;
    if (globaltimer_ns() - t0 > ab.limit_ns) {
      raise_abort(ab);
      return false;
    }
  }
}

// Eight fp32 accumulator values (bit patterns) to eight bf16, times scale.
__device__ __forceinline__ uint4 pack8_bf16(const uint32_t* y, float scale) {
  uint4 w;
  w.x = pack_bf16x2(__uint_as_float(y[0]) * scale, __uint_as_float(y[1]) * scale);
  w.y = pack_bf16x2(__uint_as_float(y[2]) * scale, __uint_as_float(y[3]) * scale);
  w.z = pack_bf16x2(__uint_as_float(y[4]) * scale, __uint_as_float(y[5]) * scale);
  w.w = pack_bf16x2(__uint_as_float(y[6]) * scale, __uint_as_float(y[7]) * scale);
  return w;
}

// One 64-column chunk of a dK or dV row (TMEM values), times scale, as bf16:
// either into row r of a 128-byte-swizzled [128 rows x 64 columns] TMA box
// (the 16-byte unit u of a row sits at u ^ (r % 8), so the eight threads of
// a store phase write eight different bank groups), or straight to global
// memory (a row of a tile cut by the end of its sequence).
__device__ __forceinline__ void chunk_to_box(uint8_t* box, const uint32_t (&x)[2][32], float scale, int r) {
  uint8_t* row = box + r * 128;
#pragma unroll
  for (int u = 0; u < 8; ++u)
    *reinterpret_cast<uint4*>(row + ((u ^ (r & 7)) << 4)) = pack8_bf16(x[u / 4] + 8 * (u % 4), scale);
}
__device__ __forceinline__ void chunk_to_global(__nv_bfloat16* dst, const uint32_t (&x)[2][32], float scale) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int u = 0; u < 8; ++u) d4[u] = pack8_bf16(x[u / 4] + 8 * (u % 4), scale);
}

// DET: deterministic dQ. Every query tile receives its dQ contributions in
// key-tile order j = 0, 1, ...: key tile j waits on the tile's counter for
// its turn, adds, waits for the addition to land and advances the counter.
// The work list is then in (sequence, key tile) order, so a key tile only
// ever waits for items claimed before it: no cycle of waits can form.
template <int D, bool CAUSAL, bool DET>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
               const __grid_constant__ CUtensorMap tm_dqacc, const BwdArgs a) {
  using L = BwdSmem<D>;
  using TC = TCols<D>;
  constexpr int NQ = L::kQStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  Bars& bars = *reinterpret_cast<Bars*>(smem + L::kBar);
  auto* hdr = reinterpret_cast<WsHeader*>(a.workspace);
  const int2* pairs = reinterpret_cast<const int2*>(static_cast<const char*>(a.workspace) + a.pairs_offset);
  const float* dvec = reinterpret_cast<const float*>(static_cast<const char*>(a.workspace) + a.dvec_offset);
  float* dqacc = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + a.dqacc_offset);
  uint32_t* qcount = reinterpret_cast<uint32_t*>(static_cast<char*>(a.workspace) + a.qcount_offset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // The layout uses the whole opt-in shared memory with no alignment slack:
  // the swizzled tiles need a 1024-byte-aligned base. The dynamic window
  // starts aligned on this architecture; if it ever did not, the call
  // reports an error instead of computing garbage.
  if ((smem_u32(smem) & 1023u) != 0) {
    griddep_wait();
    if (threadIdx.x == 0) atomicCAS(&hdr->status, 0u, static_cast<uint32_t>(FA_ERR_CUDA));
    return;
  }

  if (threadIdx.x == 0) {
    mbar_init(&bars.kv_full, 1);
    mbar_init(&bars.kv_empty, 1);
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&bars.q_full[i], 1);
      mbar_init(&bars.q_empty[i], 1);
      mbar_init(&bars.do_full[i], 1);
      mbar_init(&bars.do_empty[i], 1);
      mbar_init(&bars.ld_full[i], 2);
      mbar_init(&bars.ld_empty[i], 8);
    }
    mbar_init(&bars.s_full[0], 1);
    mbar_init(&bars.s_full[1], 1);
    mbar_init(&bars.dp_full, 1);
    mbar_init(&bars.p_full, 8);
    mbar_init(&bars.ds_full, 8);
    mbar_init(&bars.dq_full, 1);
    mbar_init(&bars.dq_free, 4);
    mbar_init(&bars.dkv_full, 1);
    mbar_init(&bars.dv_free, 4);
    mbar_init(&bars.dk_free, 4);
    mbar_init(&bars.drain, 1);
    // Item consumers: MMA warp (1), row loaders (2), P/dS warps (8), drain warps (4).
    item_ring_init(bars.items, 15);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == kDrainWarp0 && lane == 0) {
    tma_prefetch_desc(&tm_dk);
    tma_prefetch_desc(&tm_dv);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // The kernel launched behind this one may be scheduled now (it waits for
  // this grid before it touches any of its results).
  griddep_launch_dependents();
  // Everything above is local to the CTA; the work list, the inputs and the
  // outputs are touched only after the kernel before this one has finished.
  griddep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  const Abort ab{&bars.abort_flag, &hdr->status, a.wait_ns};
  const int n_pairs = static_cast<int>(hdr->n_pairs);
  const int n_items = (hdr->status == FA_OK) ? n_pairs * a.Hk : 0;
  // Class order outside the deterministic mode (whose list is in tile
  // order, and whose query tiles take their dQ turns in key-tile order).
  constexpr bool kClassOrder = !DET;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      // It claims each item ahead of time (while the previous item's last
      // Q/dO tiles are still in use), decodes it once for every role, warms
      // L2 with its K/V tiles and loads the first Q/dO tiles before waiting
      // for the K/V buffer, so an item's first step starts without an
      // exposed load.
      uint32_t m = 0, p = 0, ni = 0;
      uint32_t class_end[kCostClasses];
#pragma unroll
      for (int k = 0; k < kCostClasses; ++k) class_end[k] = kClassOrder ? hdr->class_end[k] : 0u;
      auto load_qdo = [&](const Item& it, int s) -> bool {
        const int st = p % NQ;
        const Step sp = item_step(it, s);
        const int qrow = it.s.q0 + sp.t * BM;
        uint8_t* sq = smem + L::kQdo + 2 * st * L::kQTile;
        uint8_t* sdo = sq + L::kQTile;
        const uint32_t ph = ((p / NQ) - 1) & 1;
        if (p >= NQ && !wait_bar(&bars.q_empty[st], ph, ab)) return false;
        mbar_arrive_expect_tx(&bars.q_full[st], L::kQTile);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_2d(&tm_q, &bars.q_full[st], sq + c * L::kQChunk, sp.h * D + c * 64, qrow);
        if (p >= NQ && !wait_bar(&bars.do_empty[st], ph, ab)) return false;
        mbar_arrive_expect_tx(&bars.do_full[st], L::kQTile);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_2d(&tm_do, &bars.do_full[st], sdo + c * L::kQChunk, sp.h * D + c * 64, qrow);
        ++p;
        return true;
      };
      for (;;) {
        int idx;
        Item it;
        auto decode = [&](int slot, int v) {
          it = get_item<kClassOrder>(a, pairs, v, n_pairs, class_end);
          bars.item_data[slot] = it;
        };
        if (!publish_item_decoded(bars.items, ni, &hdr->work_counter, n_items, idx, ab, decode)) goto producer_done;
        if (idx < 0) break;
        if (it.n == 0) continue;
        const int krow = it.s.k0 + it.j * BN;
        if (m > 0)
          for (int c = 0; c < L::kChunks; ++c) {
            tma_prefetch_2d(&tm_k, it.hk * D + c * 64, krow);
            tma_prefetch_2d(&tm_v, it.hk * D + c * 64, krow);
          }
        const int pre = it.n < NQ - 1 ? it.n : NQ - 1;
        int s = 0;
        for (; s < pre; ++s)
          if (!load_qdo(it, s)) goto producer_done;
        if (m > 0 && !wait_bar(&bars.kv_empty, (m - 1) & 1, ab)) goto producer_done;
        mbar_arrive_expect_tx(&bars.kv_full, 2 * L::kKTile);
        for (int c = 0; c < L::kChunks; ++c) {
          tma_load_2d(&tm_k, &bars.kv_full, smem + L::kK + c * L::kKChunk, it.hk * D + c * 64, krow);
          tma_load_2d(&tm_v, &bars.kv_full, smem + L::kV + c * L::kKChunk, it.hk * D + c * 64, krow);
        }
        ++m;
        for (; s < it.n; ++s)
          if (!load_qdo(it, s)) goto producer_done;
      }
    producer_done:
      if (m > 0) wait_bar_final(&bars.kv_full, (m - 1) & 1, ab);
      for (uint32_t i = (p > NQ ? p - NQ : 0); i < p; ++i) {
        wait_bar_final(&bars.q_full[i % NQ], (i / NQ) & 1, ab);
        wait_bar_final(&bars.do_full[i % NQ], (i / NQ) & 1, ab);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop converged; one elected lane issues each
    // group of MMAs and the commits. Per step p, in issue order (the tensor
    // pipe executes one thread's MMAs in order, so an MMA may overwrite TMEM
    // columns that earlier-issued MMAs read):
    //   S^T = K Q^T; [dQ^T of p-1 read out] dP^T = V dO^T; [P^T written]
    //   dV += P^T dO; [dS^T written] dK += dS^T Q; dQ^T = K^T dS^T.
    constexpr uint32_t kIdS = idesc_bf16_f32(BN, BM, false, false);  // S^T, dP^T: 128 x 128, K = D
    constexpr uint32_t kIdKV = idesc_bf16_f32(BN, D, false, true);   // dV, dK: 128 x D, K = 128 queries
    constexpr uint32_t kIdQ = idesc_bf16_f32(128, BM, true, true);   // dQ^T: 128 (>= D) x 128, K = 128 keys
    // At head_dim 64, dQ itself: 128 queries x 64, K = 128 keys, A = dS from
    // the dS^T buffer read M-major, B = K read N-major.
    constexpr uint32_t kIdQ64 = idesc_bf16_f32(BM, 64, true, true);
    const uint64_t k_kmaj = smem_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
    const uint64_t v_kmaj = smem_desc_sw128(smem_u32(smem + L::kV), 16, 1024);
    // At head_dim 64 the second 64-row half of M reads the first again
    // (lanes 64-127 of dQ^T are then ignored).
    const uint64_t k_mn = smem_desc_sw128(smem_u32(smem + L::kK), D == 128 ? L::kKChunk : 0, 1024);
    const uint64_t qdo_kmaj0 = smem_desc_sw128(smem_u32(smem + L::kQdo), 16, 1024);
    const uint64_t qdo_mn0 = smem_desc_sw128(smem_u32(smem + L::kQdo), L::kQChunk, 1024);
    const uint64_t ds_mn = smem_desc_sw128(smem_u32(smem + L::kDs), L::kDsHalf, 1024);
    constexpr uint64_t kQTileD = L::kQTile >> 4;  // descriptor step between Q and dO of a stage
    uint32_t m = 0, p = 0, ni = 0;
    for (;;) {
      int slot;
      const int idx = consume_item<true>(bars.items, ni, slot, ab);
      if (idx < 0) break;
      const Item it = bars.item_data[slot];
      __syncwarp();
      if (elect_one()) mbar_arrive(&bars.items.empty[slot]);
      __syncwarp();
      if (it.n == 0) continue;
      if (!wait_bar_warp(&bars.kv_full, m & 1, ab)) goto mma_done;
      tc_fence_after();
      // S^T of step pp into its buffer (waits for pp's Q tile).
      auto issue_s = [&](uint32_t pp) -> bool {
        const int qq = static_cast<int>(pp % NQ);
        if (!wait_bar_warp(&bars.q_full[qq], (pp / NQ) & 1, ab)) return false;
        tc_fence_after();
        if (elect_one()) {
          const uint64_t qk = opaque_u64(qdo_kmaj0) + static_cast<uint64_t>((2 * qq * L::kQTile) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t o = ((kk >> 2) * L::kKChunk + (kk & 3) * 32) >> 4;
            mma_ss(tmem + TC::s(pp), opaque_u64(k_kmaj) + o, qk + o, kIdS, kk > 0);
          }
          mma_commit(&bars.s_full[TC::sbar(pp)]);
        }
        __syncwarp();
        return true;
      };
      for (int s = 0; s < it.n; ++s, ++p) {
        const int qs = p % NQ;
        // Descriptors are rebuilt from opaque copies where they are used, so
        // that the compiler does not keep every offset form in registers.
        const uint64_t q_kmaj = opaque_u64(qdo_kmaj0) + static_cast<uint64_t>((2 * qs * L::kQTile) >> 4);
        const uint64_t q_mn = opaque_u64(qdo_mn0) + static_cast<uint64_t>((2 * qs * L::kQTile) >> 4);
        // With two S^T buffers an item's later steps had their S^T issued
        // during the step before.
        if ((!TC::kTwoS || s == 0) && !issue_s(p)) goto mma_done;
        // dP^T goes where the previous step's dQ^T is until the drain group
        // has read it out.
        if (p > 0 && !wait_bar_warp(&bars.dq_free, (p - 1) & 1, ab)) goto mma_done;
        if (!wait_bar_warp(&bars.do_full[qs], (p / NQ) & 1, ab)) goto mma_done;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t o = ((kk >> 2) * L::kKChunk + (kk & 3) * 32) >> 4;
            mma_ss(tmem + kColDP, opaque_u64(v_kmaj) + o, q_kmaj + kQTileD + o, kIdS, kk > 0);
          }
          mma_commit(&bars.dp_full);
        }
        __syncwarp();
        if (!wait_bar_warp(&bars.p_full, p & 1, ab)) goto mma_done;
        // First step of an item: the drain group must have read the previous
        // item's dV (then dK) out of TMEM.
        if (s == 0 && m > 0 && !wait_bar_warp(&bars.dv_free, (m - 1) & 1, ab)) goto mma_done;
        tc_fence_after();
        const uint32_t acc = s > 0 ? 1u : 0u;
        if (elect_one()) {
          // dV += P^T dO: P^T bf16 in TMEM (16 queries = 8 columns per MMA;
          // queries 64-127 start 64 columns further), dO MN-major.
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            mma_ts(tmem + TC::dv, tmem + TC::s(p) + (kk >> 2) * 64 + (kk & 3) * 8,
                   q_mn + kQTileD + ((kk * 2048) >> 4), kIdKV, (acc | kk) ? 1u : 0u);
        }
        __syncwarp();
        // The next step's S^T into the other buffer, while the P/dS warps
        // form this step's dS^T (dK below reads this step's buffer).
        if (TC::kTwoS && s + 1 < it.n && !issue_s(p + 1)) goto mma_done;
        if (!wait_bar_warp(&bars.ds_full, p & 1, ab)) goto mma_done;
        if (s == 0 && m > 0 && !wait_bar_warp(&bars.dk_free, (m - 1) & 1, ab)) goto mma_done;
        tc_fence_after();
        if (elect_one()) {
          // dK += dS^T Q (dS^T bf16 in TMEM, 32 columns after its P^T).
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            mma_ts(tmem + TC::dk, tmem + TC::s(p) + (kk >> 2) * 64 + 32 + (kk & 3) * 8, q_mn + ((kk * 2048) >> 4),
                   kIdKV, (acc | kk) ? 1u : 0u);
          // dQ^T = K^T dS^T (dS^T from shared memory) into the dP^T columns;
          // at head_dim 64 dQ = dS K instead (one query row per TMEM lane, so
          // all four drain warps read it, and N = 64 with no padded half).
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            if constexpr (D == 64)
              mma_ss(tmem + kColDP, opaque_u64(ds_mn) + ((kk * 2048) >> 4), opaque_u64(k_mn) + ((kk * 2048) >> 4),
                     kIdQ64, kk > 0);
            else
              mma_ss(tmem + kColDP, opaque_u64(k_mn) + ((kk * 2048) >> 4), opaque_u64(ds_mn) + ((kk * 2048) >> 4),
                     kIdQ, kk > 0);
          }
          mma_commit(&bars.dq_full);
        }
        __syncwarp();
      }
      if (elect_one()) {
        mma_commit(&bars.dkv_full);
        mma_commit(&bars.kv_empty);
      }
      __syncwarp();
      ++m;
    }
  mma_done:
    if (elect_one()) mma_commit(&bars.drain);
    __syncwarp();
    wait_bar_final(&bars.drain, 0, ab);
  } else if (warp < kPdsWarp0) {
    // ------------------------------------------------------------ lse / Dv rows
    // Two rows per thread (r and r + 64) of the step's 128 query rows.
    const int r = threadIdx.x - 64;
    uint32_t p = 0, ni = 0;
    for (;;) {
      int islot;
      const int idx = consume_item<true>(bars.items, ni, islot, ab);
      if (idx < 0) break;
      const Item it = bars.item_data[islot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.items.empty[islot]);
      for (int s = 0; s < it.n; ++s, ++p) {
        const int slot = p % NQ;
        if (p >= NQ && !wait_bar_warp(&bars.ld_empty[slot], ((p / NQ) - 1) & 1, ab)) goto loader_done;
        const Step sp = item_step(it, s);
        float* ld = reinterpret_cast<float*>(smem + L::kLd) + slot * 2 * BM;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int rr = r + 64 * u;
          const int qi = sp.t * BM + rr;  // row within the sequence
          // Stored negated and in base 2: -lse*log2(e); -inf for rows outside
          // the sequence or without a visible key, which makes their P exactly 0.
          float nlse2 = -INFINITY, dv = 0.f;
          if (qi < it.s.lq) {
            const size_t gq = static_cast<size_t>(it.s.q0) + qi;
            const float l = __ldg(a.lse + static_cast<size_t>(sp.h) * a.total_q + gq);
            if (l != -INFINITY) {
              nlse2 = -l * 1.4426950408889634f;
              dv = __ldg(dvec + static_cast<size_t>(sp.h) * a.tq_pad + gq);
            }
          }
          ld[rr] = nlse2;
          ld[BM + rr] = dv;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.ld_full[slot]);
      }
    }
  loader_done:;
  } else if (warp < kDrainWarp0) {
    // ------------------------------------------------------------ P^T, dS^T
    // Warpgroup qh owns queries 64*qh .. 64*qh+63 of every step; thread = key
    // row = TMEM lane. Phase 1: P^T from S^T (handed to the dV MMA at once);
    // phase 2: dS^T from dP^T and the bf16 P^T values kept in registers.
    const int qh = (warp - kPdsWarp0) >> 2;
    const int kr = (threadIdx.x - kPdsWarp0 * 32) & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_dp = tmem + lane_base + kColDP + qh * 64;  // dP^T of my queries
    uint8_t* ds_row = smem + L::kDs + qh * L::kDsHalf + kr * 128;
    uint32_t p = 0, ni = 0;
    for (;;) {
      int islot;
      const int idx = consume_item<true>(bars.items, ni, islot, ab);
      if (idx < 0) break;
      const Item it = bars.item_data[islot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.items.empty[islot]);
      const int kg = it.j * BN + kr;  // key index within the sequence
      const bool key_ok = kg < it.s.lk;
      const int diag = it.s.lk - it.s.lq;
      for (int s = 0; s < it.n; ++s, ++p) {
        const int slot = p % NQ;
        if (!wait_bar_warp(&bars.s_full[TC::sbar(p)], TC::spar(p), ab)) goto compute_done;
        const uint32_t t_s = tmem + lane_base + TC::s(p) + qh * 64;  // S^T of my queries; P^T, dS^T after it
        if (!wait_bar_warp(&bars.ld_full[slot], (p / NQ) & 1, ab)) goto compute_done;
        tc_fence_after();
        const float* ld = reinterpret_cast<const float*>(smem + L::kLd) + slot * 2 * BM + qh * 64;
        const int row0 = item_step(it, s).t * BM + qh * 64;  // first query row of my half
        // Visible iff kg <= row + diag, i.e. e >= kg - diag - row0; keys past
        // the sequence see nothing.
        int e_min = CAUSAL ? kg - diag - row0 : 0;
        if (!key_ok) e_min = 64;
        const uint64_t sc2 = f2_make(a.scale_log2, a.scale_log2);
        // P^T of my 64 queries as bf16 pairs: written to TMEM for the dV MMA
        // and kept in registers for dS^T, so that dS^T is formed from exactly
        // the probabilities the dV MMA uses.
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32];
          tmem_ld32(t_s + c * 32, sv);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int q = c * 32 + e;
            const uint64_t nl2 = *reinterpret_cast<const uint64_t*>(ld + q);
            float x0, x1;
            f2_split(f2_fma(f2_make(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, nl2), x0, x1);
            float p0 = ex2_approx(x0);
            float p1 = ex2_approx(x1);
            if (q < e_min) p0 = 0.f;
            if (q + 1 < e_min) p1 = 0.f;
            pk[q / 2] = pack_bf16x2(p0, p1);
          }
          // P^T into the first 32 columns of my S^T half; the second chunk
          // writes columns the first chunk has already read.
          tmem_st16(t_s + c * 16, *reinterpret_cast<const uint32_t(*)[16]>(&pk[c * 16]));
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full);
        // dS^T of the previous step has been read by its dQ^T MMAs: dP^T of
        // this step goes where that dQ^T was and is issued only after the
        // drain group has read it out.
        if (!wait_bar_warp(&bars.dp_full, p & 1, ab)) goto compute_done;
        tc_fence_after();
        const uint64_t* dv2p = reinterpret_cast<const uint64_t*>(ld + BM);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t dpv[32];
          tmem_ld32(t_dp + c * 32, dpv);
          tmem_wait_ld();
          uint32_t dsk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int q = c * 32 + e;
            float d0, d1;
            const uint32_t pp = pk[q / 2];  // bf16 pair -> two exact fp32 values
            f2_split(f2_mul(f2_make(__uint_as_float(pp << 16), __uint_as_float(pp & 0xffff0000u)),
                            f2_sub(f2_make(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])), dv2p[q / 2])),
                     d0, d1);
            dsk[e / 2] = pack_bf16x2(d0, d1);
          }
          // dS^T into TMEM (A operand of dK) and into shared memory, row kr,
          // queries c*32 .. c*32+31: four 16-byte units, 128-byte swizzle
          // (B operand of dQ^T).
          tmem_st16(t_s + 32 + c * 16, dsk);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int chunk = (c * 4 + u) ^ (kr & 7);
            *reinterpret_cast<uint4*>(ds_row + chunk * 16) =
                make_uint4(dsk[4 * u], dsk[4 * u + 1], dsk[4 * u + 2], dsk[4 * u + 3]);
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars.ds_full);
          mbar_arrive(&bars.ld_empty[slot]);
        }
      }
    }
  compute_done:;
  } else {
    // ------------------------------------------------------------ dQ drain, dK/dV
    const int t = threadIdx.x - kDrainWarp0 * 32;  // 0..127: TMEM lane (d for dQ^T, key row for dK/dV)
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t p = 0, m = 0, ni = 0;
    uint32_t* det_prev = nullptr;  // deterministic mode: counter whose turn is still to be passed on
    for (;;) {
      int islot;
      const int idx = consume_item<true>(bars.items, ni, islot, ab);
      // Group-uniform: this group uses named barriers, so all four warps
      // must leave together (end of work, or an abort seen by any warp).
      if (!named_bar_and(1, 128, idx >= 0)) break;
      const Item it = bars.item_data[islot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.items.empty[islot]);
      const int kg = it.j * BN + t;
      const bool key_ok = kg < it.s.lk;
      const size_t krow = (static_cast<size_t>(it.s.k0) + kg) * a.Hk + it.hk;
      if (it.n == 0) {
        if (key_ok) {
          uint4* dk = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.dk) + krow * D);
          uint4* dv = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.dv) + krow * D);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) dk[c] = dv[c] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      int qs = 0;  // Q/dO stage of the current step: its staging area
      for (int s = 0; s < it.n; ++s, ++p) {
        // Group-wide decision: every warp of this group reaches the vote, so
        // none is left waiting on the named barriers below.
        if (!named_bar_and(1, 128, wait_bar(&bars.dq_full, p & 1, ab))) goto drain_done;
        tc_fence_after();
        // Every MMA of the step has completed, so its Q/dO stage is free:
        // the step's fp32 dQ tile (128 x D) is staged there, queries 0-63
        // over the Q half and 64-127 over the dO half (128 consecutive rows
        // of one head are one contiguous block of the head-major
        // accumulator). Each half leaves with its own bulk reduction as soon
        // as it is staged, and the Q half goes back to the loader once its
        // reduction has read it, so the next Q tile loads while the second
        // half is still being reduced. The deterministic mode adds the whole
        // tile at once, in its query tile's turn.
        qs = static_cast<int>(p % NQ);
        float* stage = reinterpret_cast<float*>(smem + L::kQdo + 2 * qs * L::kQTile);
        const Step sp = item_step(it, s);
        const size_t q0 = static_cast<size_t>(it.s.q0) + static_cast<size_t>(sp.t) * BM;
        uint32_t* cnt = qcount + static_cast<size_t>(sp.h) * a.tq_pad + q0;
        float* gdq = dqacc + (static_cast<size_t>(sp.h) * a.tq_pad + q0) * D;
        if constexpr (D == 64) {
          // Thread t holds query row t of dQ (64 channels): one read frees
          // the columns at once. The row is staged as two 128-byte-swizzled
          // boxes of [128 rows x 32 channels] (channels 0-31 over the Q half
          // of the stage, 32-63 over the dO half; the swizzle spreads a
          // warp's stores over all banks) and leaves with two tensor
          // reductions into the accumulator viewed as [H * tq_pad, 64].
          uint32_t v[64];
          tmem_ld32(tmem + lane_base + kColDP, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          tmem_ld32(tmem + lane_base + kColDP + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.dq_free);
          uint8_t* st8 = reinterpret_cast<uint8_t*>(stage) + t * 128;
#pragma unroll
          for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(st8 + b * L::kQTile + ((c ^ (t & 7)) << 4)) =
                  make_uint4(v[32 * b + 4 * c], v[32 * b + 4 * c + 1], v[32 * b + 4 * c + 2], v[32 * b + 4 * c + 3]);
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (t == 0) {
            const int y = sp.h * a.tq_pad + static_cast<int>(q0);
            if (DET) wait_dq_turn(cnt, static_cast<uint32_t>(it.j), ab);
            if (!*ab.flag) {
              if (DET) fence_proxy_async_global();
              tma_reduce_add_2d(&tm_dqacc, stage, 0, y);
              if (!DET) bulk_commit_group();
              tma_reduce_add_2d(&tm_dqacc, reinterpret_cast<uint8_t*>(stage) + L::kQTile, 32, y);
              bulk_commit_group();
              if (DET) {
                if (det_prev) {
                  bulk_wait_group1();
                  fence_proxy_async_global();
                  st_release_gpu(det_prev, static_cast<uint32_t>(it.j) + 1u);
                }
                det_prev = cnt;
              }
            }
          }
        } else {
  #pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            uint32_t v0[32], v1[32];
            tmem_ld32(tmem + lane_base + kColDP + h * 64, v0);
            tmem_ld32(tmem + lane_base + kColDP + h * 64 + 32, v1);
            tmem_wait_ld();
            if (h == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bars.dq_free);
            }
            float* st = stage + h * 64 * D;
            if (t < D) {
  #pragma unroll
              for (int e = 0; e < 32; ++e) st[e * D + t] = __uint_as_float(v0[e]);
  #pragma unroll
              for (int e = 0; e < 32; ++e) st[(32 + e) * D + t] = __uint_as_float(v1[e]);
            }
            if (!DET) {
              fence_proxy_async_smem();
              named_bar_sync(1, 128);
              if (t == 0 && !*ab.flag) {
                bulk_reduce_add_f32(gdq + h * 64 * D, st, 64 * D * 4);
                bulk_commit_group();
              }
            }
          }
          if (DET) {
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (t == 0) {
              // This query tile's turn first (a wait that runs out raises the
              // abort flag, and nothing more is added).
              wait_dq_turn(cnt, static_cast<uint32_t>(it.j), ab);
              if (!*ab.flag) {
                fence_proxy_async_global();
                bulk_reduce_add_f32(gdq, stage, BM * D * 4);
                bulk_commit_group();
                // Pass the previous step's turn on once its addition has been
                // performed (it was issued a step ago, so this rarely waits);
                // this step's turn passes on at the next step or item end.
                if (det_prev) {
                  bulk_wait_group1();
                  fence_proxy_async_global();
                  st_release_gpu(det_prev, static_cast<uint32_t>(it.j) + 1u);
                }
                det_prev = cnt;
              }
            }
          }
        }
        // Hand the stage back to the loader half by half once the reductions
        // have read it (an item's last stage serves the dK/dV stores first).
        if (t == 0 && s + 1 < it.n) {
          if (DET)
            bulk_wait_group_read0();
          else
            bulk_wait_group_read1();
          mbar_arrive(&bars.q_empty[qs]);
          bulk_wait_group_read0();
          mbar_arrive(&bars.do_empty[qs]);
        }
      }
      if (DET && t == 0 && det_prev) {
        bulk_wait_group0();
        fence_proxy_async_global();
        st_release_gpu(det_prev, static_cast<uint32_t>(it.j) + 1u);
        det_prev = nullptr;
      }
      // dK, dV of this key tile. dV is read out of TMEM first and released
      // at once, so the next item's first dV MMAs wait only for that read;
      // dK follows. A whole tile leaves through TMA stores from the last
      // step's stage (the coalesced path, which keeps the load/store unit
      // free for the P/dS warps): dV in its first half, dK in its second; a
      // tile cut by the end of its sequence is stored row by row, so that no
      // row of the next sequence is touched.
      if (!named_bar_and(1, 128, wait_bar(&bars.dkv_full, m & 1, ab))) goto drain_done;
      tc_fence_after();
      {
        const bool whole = (it.j + 1) * BN <= it.s.lk;  // the same for the whole group
        const int row0 = it.s.k0 + it.j * BN;
        uint8_t* stage = smem + L::kQdo + 2 * qs * L::kQTile;
        if (whole) {
          // The last dQ reduction must have read the stage.
          if (t == 0) bulk_wait_group_read0();
          named_bar_sync(1, 128);
        }
#pragma unroll 1
        for (int g = 0; g < 2; ++g) {  // g = 0: dV, g = 1: dK (times scale)
          const int col = g == 0 ? TC::dv : TC::dk;
          const float sc = g == 0 ? 1.f : a.scale;
          __nv_bfloat16* gdst = static_cast<__nv_bfloat16*>(g == 0 ? a.dv : a.dk) + krow * D;
          uint8_t* box = stage + g * L::kQTile;  // bf16 boxes of [128 rows x 64 columns], 16 KB apart
#pragma unroll 1
          for (int c = 0; c < D / 64; ++c) {
            uint32_t x[2][32];
            tmem_ld32(tmem + lane_base + col + c * 64, x[0]);
            tmem_ld32(tmem + lane_base + col + c * 64 + 32, x[1]);
            tmem_wait_ld();
            if (c == D / 64 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(g == 0 ? &bars.dv_free : &bars.dk_free);
            }
            if (whole)
              chunk_to_box(box + c * 16384, x, sc, t);
            else if (key_ok)
              chunk_to_global(gdst + c * 64, x, sc);
          }
          if (whole) {
            fence_proxy_async_smem();
            named_bar_sync(1, 128);
            if (t == 0) {
              const CUtensorMap* map = g == 0 ? &tm_dv : &tm_dk;
#pragma unroll
              for (int c = 0; c < D / 64; ++c) tma_store_2d(map, box + c * 16384, it.hk * D + c * 64, row0);
              bulk_commit_group();
            }
          }
        }
        if (t == 0) {
          bulk_wait_group_read0();  // the stores (and the last reduction) have read the stage
          mbar_arrive(&bars.q_empty[qs]);
          mbar_arrive(&bars.do_empty[qs]);
        }
      }
      ++m;
    }
  drain_done:
    // Bulk operations still reading shared memory must finish before exit.
    if (t == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// The two streaming kernels around the main one take kUnits (row, head)
// units per warp, consecutive in memory, and issue all their loads before
// using any, so that enough bytes are in flight to run at HBM speed. They
// serve every head dimension (64, 128, 256): lane l of a warp handles
// elements l*E .. l*E+E-1 of a row of D = 32*E.
constexpr int kUnits = 4;

template <int N>
struct Words;  // N 32-bit words in one vector access
template <>
struct Words<1> {
  using T = uint32_t;
};
template <>
struct Words<2> {
  using T = uint2;
};
template <>
struct Words<4> {
  using T = uint4;
};

// Dv[h, r] = sum_c dO[r, h, c] * O[r, h, c] in fp32, and dQacc[h, r, :] = 0.
template <int D>
__device__ __forceinline__ void preprocess_rows(const BwdArgs& a) {
  constexpr int E = D / 32;  // bf16 elements per lane: 2, 4 or 8 (4, 8 or 16 bytes)
  using V = typename Words<E / 2>::T;
  const long long units = static_cast<long long>(a.total_q) * a.H;
  const long long u0 = ((static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * kUnits;
  const int lane = threadIdx.x & 31;
  if (u0 >= units) return;
  const V* o = reinterpret_cast<const V*>(static_cast<const __nv_bfloat16*>(a.out) + u0 * D) + lane;
  const V* g = reinterpret_cast<const V*>(static_cast<const __nv_bfloat16*>(a.dout) + u0 * D) + lane;
  V ov[kUnits], gv[kUnits];
#pragma unroll
  for (int i = 0; i < kUnits; ++i) {
    if (u0 + i < units) {
      ov[i] = o[i * 32];
      gv[i] = g[i * 32];
    } else {
      ov[i] = V{};
      gv[i] = V{};
    }
  }
  float acc[kUnits];
#pragma unroll
  for (int i = 0; i < kUnits; ++i) {
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov[i]);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv[i]);
    acc[i] = 0.f;
#pragma unroll
    for (int k = 0; k < E / 2; ++k) {
      const float2 x = __bfloat1622float2(o2[k]), y = __bfloat1622float2(g2[k]);
      acc[i] = fmaf(x.x, y.x, acc[i]);
      acc[i] = fmaf(x.y, y.y, acc[i]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1)
#pragma unroll
    for (int i = 0; i < kUnits; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
  float* dvec = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + a.dvec_offset);
  float* dqacc = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + a.dqacc_offset);
  uint32_t* qcount = reinterpret_cast<uint32_t*>(static_cast<char*>(a.workspace) + a.qcount_offset);
#pragma unroll
  for (int i = 0; i < kUnits; ++i) {
    const long long u = u0 + i;
    if (u >= units) break;
    const int row = static_cast<int>(u / a.H), h = static_cast<int>(u % a.H);
    const size_t hr = static_cast<size_t>(h) * a.tq_pad + row;
    if (lane == 0) {
      dvec[hr] = acc[i];
      qcount[hr] = 0u;
    }
    float4* z = reinterpret_cast<float4*>(dqacc + hr * D);
    for (int c = lane; c < D / 4; c += 32) z[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// Reads only the caller's tensors and writes only its own workspace regions,
// so it runs while the work-list kernel before it is still working; it waits
// for that kernel before it exits, so that its own completion, which the
// main kernel waits for, implies the work list's.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const BwdArgs a) {
  griddep_launch_dependents();
  preprocess_rows<D>(a);
  griddep_wait();
}

// dQ[r, h, :] = bf16(scale * dQacc[h, r, :]).
template <int D>
__global__ void __launch_bounds__(256) bwd_convert_kernel(const BwdArgs a) {
  griddep_wait();  // the accumulator comes from the main kernel before this one
  constexpr int E = D / 32;          // fp32 elements per lane: 2, 4 or 8
  constexpr int W = E < 4 ? E : 4;   // words per vector load
  constexpr int NL = E / W;          // vector loads per lane and unit
  using F = typename Words<W>::T;
  using O = typename Words<E / 2>::T;
  const long long units = static_cast<long long>(a.total_q) * a.H;
  const long long u0 = ((static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * kUnits;
  const int lane = threadIdx.x & 31;
  if (u0 >= units) return;
  const float* acc = reinterpret_cast<const float*>(static_cast<const char*>(a.workspace) + a.dqacc_offset);
  F v[kUnits][NL];
#pragma unroll
  for (int i = 0; i < kUnits; ++i) {
    const long long u = u0 + i;
    const int row = static_cast<int>(u / a.H), h = static_cast<int>(u % a.H);
    const F* src = reinterpret_cast<const F*>(acc + (static_cast<size_t>(h) * a.tq_pad + row) * D) + lane * NL;
#pragma unroll
    for (int l = 0; l < NL; ++l) v[i][l] = u < units ? src[l] : F{};
  }
#pragma unroll
  for (int i = 0; i < kUnits; ++i) {
    const long long u = u0 + i;
    if (u >= units) break;
    const float* x = reinterpret_cast<const float*>(&v[i][0]);
    O o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int k = 0; k < E / 2; ++k) ow[k] = pack_bf16x2(x[2 * k] * a.scale, x[2 * k + 1] * a.scale);
    reinterpret_cast<O*>(static_cast<__nv_bfloat16*>(a.dq) + u * D)[lane] = o;
  }
}

template <int D, bool CAUSAL, bool DET>
cudaError_t launch_main(const BwdArgs& a, const BwdMaps& m, cudaStream_t stream) {
  using L = BwdSmem<D>;
  using TC = TCols<D>;
  auto kern = bwd_kernel<D, CAUSAL, DET>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, a.grid, kThreads, L::kBytes, stream, a.chained != 0, m.q, m.k, m.v, m.dout, m.dk, m.dv,
                       m.dqacc, a);
}

}  // namespace

cudaError_t launch_bwd_preprocess(const BwdArgs& a, cudaStream_t stream) {
  const long long warps = (static_cast<long long>(a.total_q) * a.H + kUnits - 1) / kUnits;
  const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
  if (blocks == 0) return cudaSuccess;
  auto kern = a.D == 64 ? bwd_preprocess_kernel<64> : a.D == 128 ? bwd_preprocess_kernel<128> : bwd_preprocess_kernel<256>;
  return launch_kernel(kern, blocks, 256, 0, stream, a.chained != 0, a);
}

template <bool DET>
cudaError_t launch_main_det(const BwdArgs& a, const BwdMaps& m, cudaStream_t stream) {
  if (a.D == 64)
    return a.causal ? launch_main<64, true, DET>(a, m, stream) : launch_main<64, false, DET>(a, m, stream);
  return a.causal ? launch_main<128, true, DET>(a, m, stream) : launch_main<128, false, DET>(a, m, stream);
}

cudaError_t launch_bwd_main(const BwdArgs& a, const BwdMaps& m, cudaStream_t stream) {
  return a.deterministic ? launch_main_det<true>(a, m, stream) : launch_main_det<false>(a, m, stream);
}

cudaError_t launch_bwd_convert(const BwdArgs& a, cudaStream_t stream) {
  const long long warps = (static_cast<long long>(a.total_q) * a.H + kUnits - 1) / kUnits;
  const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
  if (blocks == 0) return cudaSuccess;
  auto kern = a.D == 64 ? bwd_convert_kernel<64> : a.D == 128 ? bwd_convert_kernel<128> : bwd_convert_kernel<256>;
  return launch_kernel(kern, blocks, 256, 0, stream, a.chained != 0, a);
}

}  // namespace fa
