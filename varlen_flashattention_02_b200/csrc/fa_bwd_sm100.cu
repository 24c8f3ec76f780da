// fa_bwd_sm100.cu -- backward varlen attention for sm_100a.
//
// Three kernels per call, after the work-list preparation (key-tile mode):
//  1. preprocess: Dv_i = sum_c dO_ic * O_ic (fp32, [H, rows]) and zero the
//     fp32 dQ accumulator;
//  2. main: one persistent CTA per SM takes (sequence, key/value head,
//     key-tile) items, longest first, from a global counter. For 128 keys
//     K_j, V_j of one key/value head it loops over the query heads that read
//     that head (one, or a group under grouped-query attention) and the
//     64-row query tiles that see the keys, recomputing the probabilities
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
// B200 design: persistent longest-first scheduling; warp specialisation
// (warp 0 TMA, warp 1 MMA issue, warps 2-3 stage logsumexp/Dv rows,
// warps 4-7 compute P^T and dS^T with one thread per key row, warps 8-11
// drain dQ^T from TMEM into bulk fp32 reductions and write dK/dV); dK, dV
// and the per-step S^T, dP^T tiles live in TMEM (S^T and dP^T double-
// buffered so the next step's QK^T overlaps this step's softmax); P^T goes
// back to TMEM as bf16 and feeds the dV MMA directly; dS^T is written once to
// shared memory in a layout that serves both the dK MMA (K-major A) and the
// dQ^T MMA (MN-major B).
#include <type_traits>

#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {
namespace {

constexpr int BN = kBwdBN;  // keys per item
constexpr int BM = kBwdBM;  // queries per step
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr int kColDK = 0, kColDV = 128, kColS = 256, kColDP = 384;  // TMEM column map

template <int D>
struct BwdSmem {
  static constexpr int kQStages = 3;  // Q/dO stages (and logsumexp/Dv slots) in flight
  static constexpr int kChunks = D / 64;
  static constexpr int kKChunk = BN * 128;  // [128 rows x 64 bf16] swizzled chunk
  static constexpr int kQChunk = BM * 128;  // [ 64 rows x 64 bf16]
  static constexpr int kKTile = kChunks * kKChunk;
  static constexpr int kQTile = kChunks * kQChunk;
  static constexpr int kDsTile = BN * BM * 2;  // dS^T [128 keys x 64 queries] bf16
  static constexpr int kK = 0;
  static constexpr int kV = kK + kKTile;
  static constexpr int kQdo = kV + kKTile;  // stage s: Q at kQdo + 2s*QTile, dO after it
  static constexpr int kDs = kQdo + 2 * kQStages * kQTile;
  static constexpr int kStage = kDs + 2 * kDsTile;   // fp32 dQ [64 x D]
  static constexpr int kLd = kStage + BM * D * 4;    // kQStages slots x (lse[64], dv[64]) fp32
  static constexpr int kBar = kLd + kQStages * 2 * BM * 4;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;
};

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

__device__ __forceinline__ Item get_item(const BwdArgs& a, const int2* pairs, int idx) {
  Item it;
  const int2 pr = pairs[idx / a.Hk];
  it.hk = idx % a.Hk;
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
  uint64_t qdo_full[3], qdo_empty[3];
  uint64_t st_full[2];
  uint64_t ds_full[2], ds_empty[2];
  uint64_t dq_full[2], dq_empty[2];
  uint64_t dkv_full, dv_empty, dk_empty;
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

// One row of D accumulator values to bf16 in global memory, times scale.
template <int D>
__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, const uint32_t (&x)[D / 32][32], float scale) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int e = 0; e < D / 8; ++e) d4[e] = pack8_bf16(x[e / 4] + 8 * (e % 4), scale);
}

// Row r of a [128 x D] bf16 tile into shared memory in the layout of the
// 128-byte-swizzled TMA boxes (64 columns x 128 rows per box, box c at
// c * 16 KB, 1024-byte aligned): the 16-byte unit u of a 128-byte row sits
// at position u ^ (r % 8). The eight threads of a store phase therefore
// write eight different bank groups.
template <int D>
__device__ __forceinline__ void stage_row_sw128(uint8_t* tile, const uint32_t (&x)[D / 32][32], float scale, int r) {
  uint8_t* row = tile + r * 128;
#pragma unroll
  for (int e = 0; e < D / 8; ++e) {
    const int c = e / 8, u = e % 8;
    *reinterpret_cast<uint4*>(row + c * 16384 + ((u ^ (r & 7)) << 4)) = pack8_bf16(x[e / 4] + 8 * (e % 4), scale);
  }
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
               const BwdArgs a) {
  using L = BwdSmem<D>;
  constexpr int NQ = L::kQStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(smem + L::kBar);
  auto* hdr = reinterpret_cast<WsHeader*>(a.workspace);
  const int2* pairs = reinterpret_cast<const int2*>(static_cast<const char*>(a.workspace) + a.pairs_offset);
  const float* dvec = reinterpret_cast<const float*>(static_cast<const char*>(a.workspace) + a.dvec_offset);
  float* dqacc = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + a.dqacc_offset);
  uint32_t* qcount = reinterpret_cast<uint32_t*>(static_cast<char*>(a.workspace) + a.qcount_offset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars.kv_full, 1);
    mbar_init(&bars.kv_empty, 1);
    for (int i = 0; i < L::kQStages; ++i) {
      mbar_init(&bars.qdo_full[i], 1);
      mbar_init(&bars.qdo_empty[i], 1);
      mbar_init(&bars.ld_full[i], 2);
      mbar_init(&bars.ld_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.st_full[i], 1);
      mbar_init(&bars.ds_full[i], 4);
      mbar_init(&bars.ds_empty[i], 1);
      mbar_init(&bars.dq_full[i], 1);
      mbar_init(&bars.dq_empty[i], 4);
    }
    mbar_init(&bars.dkv_full, 1);
    mbar_init(&bars.dv_empty, 4);
    mbar_init(&bars.dk_empty, 4);
    mbar_init(&bars.drain, 1);
    // Item consumers: MMA warp (1), row loaders (2), P/dS warps (4), drain warps (4).
    item_ring_init(bars.items, 11);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_dk);
    tma_prefetch_desc(&tm_dv);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  const Abort ab{&bars.abort_flag, &hdr->status, a.wait_ns};
  const int n_items = (hdr->status == FA_OK) ? static_cast<int>(hdr->n_pairs) * a.Hk : 0;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      // It claims each item ahead of time (while the previous item's last
      // Q/dO tiles are still in use), decodes it once for every role, warms
      // L2 with its K/V tiles and loads the first Q/dO tiles before waiting
      // for the K/V buffer, so an item's first step starts without an
      // exposed load.
      uint32_t m = 0, p = 0, ni = 0;
      auto load_qdo = [&](const Item& it, int s) -> bool {
        const int st = p % NQ;
        if (p >= NQ && !wait_bar(&bars.qdo_empty[st], ((p / NQ) - 1) & 1, ab)) return false;
        const Step sp = item_step(it, s);
        const int qrow = it.s.q0 + sp.t * BM;
        uint8_t* sq = smem + L::kQdo + 2 * st * L::kQTile;
        uint8_t* sdo = sq + L::kQTile;
        mbar_arrive_expect_tx(&bars.qdo_full[st], 2 * L::kQTile);
        for (int c = 0; c < L::kChunks; ++c) {
          tma_load_2d(&tm_q, &bars.qdo_full[st], sq + c * L::kQChunk, sp.h * D + c * 64, qrow);
          tma_load_2d(&tm_do, &bars.qdo_full[st], sdo + c * L::kQChunk, sp.h * D + c * 64, qrow);
        }
        ++p;
        return true;
      };
      for (;;) {
        int idx;
        Item it;
        auto decode = [&](int slot, int v) {
          it = get_item(a, pairs, v);
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
      for (uint32_t i = (p > NQ ? p - NQ : 0); i < p; ++i) wait_bar_final(&bars.qdo_full[i % NQ], (i / NQ) & 1, ab);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop converged; one elected lane issues each
    // group of MMAs and the commits. Descriptors are built once and advanced
    // by constant offsets.
    constexpr uint32_t kIdS = idesc_bf16_f32(BN, BM, false, false);   // S^T, dP^T: 128 x 64, K = D
    constexpr uint32_t kIdKV = idesc_bf16_f32(BN, D, false, true);    // dV, dK: 128 x D, K = 64
    constexpr uint32_t kIdQ = idesc_bf16_f32(128, BM, true, true);    // dQ^T: 128 (>= D) x 64, K = 128
    const uint64_t k_kmaj = smem_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
    const uint64_t v_kmaj = smem_desc_sw128(smem_u32(smem + L::kV), 16, 1024);
    const uint64_t k_mn = smem_desc_sw128(smem_u32(smem + L::kK), D == 128 ? L::kKChunk : 0, 1024);
    const uint64_t qdo_kmaj0 = smem_desc_sw128(smem_u32(smem + L::kQdo), 16, 1024);
    const uint64_t qdo_mn0 = smem_desc_sw128(smem_u32(smem + L::kQdo), L::kQChunk, 1024);
    const uint64_t ds_kmaj0 = smem_desc_sw128(smem_u32(smem + L::kDs), 16, 1024);
    const uint64_t ds_mn0 = smem_desc_sw128(smem_u32(smem + L::kDs), 0, 1024);
    constexpr uint64_t kQTileD = L::kQTile >> 4;    // descriptor step between Q and dO of a stage
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
      for (int s = 0; s <= it.n; ++s) {
        if (s < it.n) {
          const uint32_t ps = p + s;
          const int st = ps & 1;      // TMEM S^T / dP^T buffer
          const int qs = ps % NQ;     // Q/dO stage
          if (!wait_bar_warp(&bars.qdo_full[qs], (ps / NQ) & 1, ab)) goto mma_done;
          if (ps >= 2 && !wait_bar_warp(&bars.dq_empty[st], ((ps >> 1) - 1) & 1, ab)) goto mma_done;
          tc_fence_after();
          const uint64_t q_desc = qdo_kmaj0 + static_cast<uint64_t>((2 * qs * L::kQTile) >> 4);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t oa = ((kk >> 2) * L::kKChunk + (kk & 3) * 32) >> 4;
              const uint64_t ob = ((kk >> 2) * L::kQChunk + (kk & 3) * 32) >> 4;
              mma_ss(tmem + kColS + st * BM, k_kmaj + oa, q_desc + ob, kIdS, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t oa = ((kk >> 2) * L::kKChunk + (kk & 3) * 32) >> 4;
              const uint64_t ob = ((kk >> 2) * L::kQChunk + (kk & 3) * 32) >> 4;
              mma_ss(tmem + kColDP + st * BM, v_kmaj + oa, q_desc + kQTileD + ob, kIdS, kk > 0);
            }
            mma_commit(&bars.st_full[st]);
          }
          __syncwarp();
        }
        if (s > 0) {
          const uint32_t pp = p + s - 1;
          const int pb = pp & 1;
          const int qs = pp % NQ;
          if (!wait_bar_warp(&bars.ds_full[pb], (pp >> 1) & 1, ab)) goto mma_done;
          // First step of an item: the drain group must have read the
          // previous item's dV (then dK) out of TMEM.
          if (s == 1 && m > 0 && !wait_bar_warp(&bars.dv_empty, (m - 1) & 1, ab)) goto mma_done;
          tc_fence_after();
          const uint64_t q_mn = qdo_mn0 + static_cast<uint64_t>((2 * qs * L::kQTile) >> 4);
          const uint64_t ds_k = ds_kmaj0 + static_cast<uint64_t>((pb * L::kDsTile) >> 4);
          const uint64_t ds_mn = ds_mn0 + static_cast<uint64_t>((pb * L::kDsTile) >> 4);
          const uint32_t acc = (s > 1) ? 1u : 0u;
          if (elect_one()) {
            // dV += P^T dO (P^T from TMEM, dO MN-major); dK += dS^T Q.
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              mma_ts(tmem + kColDV, tmem + kColS + pb * BM + kk * 8, q_mn + kQTileD + ((kk * 2048) >> 4), kIdKV,
                     (acc | kk) ? 1u : 0u);
          }
          __syncwarp();
          if (s == 1 && m > 0 && !wait_bar_warp(&bars.dk_empty, (m - 1) & 1, ab)) goto mma_done;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BM / 16; ++kk)
              mma_ss(tmem + kColDK, ds_k + ((kk * 32) >> 4), q_mn + ((kk * 2048) >> 4), kIdKV, (acc | kk) ? 1u : 0u);
            // dQ^T = K^T dS^T into the dP^T columns of this step.
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              mma_ss(tmem + kColDP + pb * BM, k_mn + ((kk * 2048) >> 4), ds_mn + ((kk * 2048) >> 4), kIdQ, kk > 0);
            mma_commit(&bars.dq_full[pb]);
            mma_commit(&bars.qdo_empty[qs]);
            mma_commit(&bars.ds_empty[pb]);
          }
          __syncwarp();
        }
      }
      if (elect_one()) {
        mma_commit(&bars.dkv_full);
        mma_commit(&bars.kv_empty);
      }
      __syncwarp();
      p += it.n;
      ++m;
    }
  mma_done:
    if (elect_one()) mma_commit(&bars.drain);
    __syncwarp();
    wait_bar_final(&bars.drain, 0, ab);
  } else if (warp < 4) {
    // ------------------------------------------------------------ lse / Dv rows
    const int r = threadIdx.x - 64;  // query row within the tile, 0..63
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
        const int qi = sp.t * BM + r;  // row within the sequence
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
        float* ld = reinterpret_cast<float*>(smem + L::kLd) + slot * 2 * BM;
        ld[r] = nlse2;
        ld[BM + r] = dv;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.ld_full[slot]);
      }
    }
  loader_done:;
  } else if (warp < 8) {
    // ------------------------------------------------------------ P^T, dS^T
    const int kr = threadIdx.x - 128;  // key row in the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
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
        const int pb = p & 1;
        if (!wait_bar_warp(&bars.st_full[pb], (p >> 1) & 1, ab)) goto compute_done;
        const int slot = p % NQ;
        if (!wait_bar_warp(&bars.ld_full[slot], (p / NQ) & 1, ab)) goto compute_done;
        if (p >= 2 && !wait_bar_warp(&bars.ds_empty[pb], ((p >> 1) - 1) & 1, ab)) goto compute_done;
        tc_fence_after();
        const float* ld = reinterpret_cast<const float*>(smem + L::kLd) + slot * 2 * BM;
        const int row0 = item_step(it, s).t * BM;  // first query row of the step
        // Visible iff kg <= row + diag, i.e. e >= kg - diag - row0; keys past
        // the sequence see nothing.
        int e_min = CAUSAL ? kg - diag - row0 : 0;
        if (!key_ok) e_min = BM;
        uint8_t* ds_row = smem + L::kDs + pb * L::kDsTile + kr * 128;
        const uint64_t sc2 = f2_make(a.scale_log2, a.scale_log2);
#pragma unroll
        for (int c = 0; c < BM / 32; ++c) {
          uint32_t sv[32], dpv[32];
          tmem_ld32(tmem + lane_base + kColS + pb * BM + c * 32, sv);
          tmem_ld32(tmem + lane_base + kColDP + pb * BM + c * 32, dpv);
          tmem_wait_ld();
          uint32_t pk[16], dsk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int q = c * 32 + e;
            // Pairs of query columns share packed f32x2 arithmetic.
            const uint64_t nl2 = *reinterpret_cast<const uint64_t*>(ld + q);
            const uint64_t dv2 = *reinterpret_cast<const uint64_t*>(ld + BM + q);
            float x0, x1;
            f2_split(f2_fma(f2_make(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, nl2), x0, x1);
            float p0 = ex2_approx(x0);
            float p1 = ex2_approx(x1);
            if (q < e_min) p0 = 0.f;
            if (q + 1 < e_min) p1 = 0.f;
            const uint64_t p2 = f2_make(p0, p1);
            float d0, d1;
            f2_split(f2_mul(p2, f2_sub(f2_make(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])), dv2)), d0, d1);
            pk[e / 2] = pack_bf16x2(p0, p1);
            dsk[e / 2] = pack_bf16x2(d0, d1);
          }
          // P^T (bf16 pairs) into the first 32 columns of this step's S^T.
          tmem_st16(tmem + lane_base + kColS + pb * BM + c * 16, pk);
          // dS^T row kr, queries c*32 .. c*32+31: four 16-byte chunks, 128-byte swizzle.
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
          mbar_arrive(&bars.ds_full[pb]);
          mbar_arrive(&bars.ld_empty[slot]);
        }
      }
    }
  compute_done:;
  } else {
    // ------------------------------------------------------------ dQ drain, dK/dV
    const int t = threadIdx.x - 256;  // 0..127: TMEM lane (d for dQ^T, key row for dK/dV)
    const int q4 = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    float* stage = reinterpret_cast<float*>(smem + L::kStage);
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
      for (int s = 0; s < it.n; ++s, ++p) {
        const int pb = p & 1;
        // Group-wide decision: every warp of this group reaches the vote, so
        // none is left waiting on the named barriers below.
        if (!named_bar_and(1, 128, wait_bar(&bars.dq_full[pb], (p >> 1) & 1, ab))) goto drain_done;
        tc_fence_after();
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem + lane_base + kColDP + pb * BM, v0);
        tmem_ld32(tmem + lane_base + kColDP + pb * BM + 32, v1);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.dq_empty[pb]);
        // The previous bulk reduction must have finished reading the stage.
        if (t == 0) bulk_wait_group_read0();
        named_bar_sync(1, 128);
        if (t < D) {
#pragma unroll
          for (int e = 0; e < 32; ++e) stage[e * D + t] = __uint_as_float(v0[e]);
#pragma unroll
          for (int e = 0; e < 32; ++e) stage[(32 + e) * D + t] = __uint_as_float(v1[e]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (t == 0) {
          const Step sp = item_step(it, s);
          const size_t q0 = static_cast<size_t>(it.s.q0) + static_cast<size_t>(sp.t) * BM;
          uint32_t* cnt = qcount + static_cast<size_t>(sp.h) * a.tq_pad + q0;
          const bool turn = !DET || wait_dq_turn(cnt, static_cast<uint32_t>(it.j), ab);
          if (turn) {
            if (DET) fence_proxy_async_global();
            bulk_reduce_add_f32(dqacc + (static_cast<size_t>(sp.h) * a.tq_pad + q0) * D, stage, BM * D * 4);
            bulk_commit_group();
            if (DET) {
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
      if (DET && t == 0 && det_prev) {
        bulk_wait_group0();
        fence_proxy_async_global();
        st_release_gpu(det_prev, static_cast<uint32_t>(it.j) + 1u);
        det_prev = nullptr;
      }
      // dK, dV of this key tile. dV is read out of TMEM first and released
      // at once, so the next item's first dV MMAs wait only for that read;
      // dK follows. A whole tile leaves through TMA stores from the stage
      // (the coalesced path, which keeps the load/store unit free for the
      // P/dS warps); a tile cut by the end of its sequence is stored row by
      // row, so that no row of the next sequence is touched.
      if (!named_bar_and(1, 128, wait_bar(&bars.dkv_full, m & 1, ab))) goto drain_done;
      tc_fence_after();
      {
        const bool whole = (it.j + 1) * BN <= it.s.lk;  // the same for the whole group
        const int row0 = it.s.k0 + it.j * BN;
        uint8_t* tile = smem + L::kStage;
        uint32_t x[D / 32][32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(tmem + lane_base + kColDV + c * 32, x[c]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.dv_empty);
        if (whole) {
          if (t == 0) bulk_wait_group_read0();  // the last dQ reduction has read the stage
          named_bar_sync(1, 128);
          stage_row_sw128<D>(tile, x, 1.f, t);
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (t == 0) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tma_store_2d(&tm_dv, tile + c * 16384, it.hk * D + c * 64, row0);
            bulk_commit_group();
          }
        } else if (key_ok) {
          store_row_bf16<D>(static_cast<__nv_bfloat16*>(a.dv) + krow * D, x, 1.f);
        }
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(tmem + lane_base + kColDK + c * 32, x[c]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.dk_empty);
        if (whole) {
          if (t == 0) bulk_wait_group_read0();  // the dV stores have read the stage
          named_bar_sync(1, 128);
          stage_row_sw128<D>(tile, x, a.scale, t);
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (t == 0) {
#pragma unroll
            for (int c = 0; c < D / 64; ++c) tma_store_2d(&tm_dk, tile + c * 16384, it.hk * D + c * 64, row0);
            bulk_commit_group();
          }
        } else if (key_ok) {
          store_row_bf16<D>(static_cast<__nv_bfloat16*>(a.dk) + krow * D, x, a.scale);
        }
      }
      ++m;
    }
  drain_done:
    // Bulk reductions still reading the stage must finish before exit.
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
// using any, so that enough bytes are in flight to run at HBM speed.
constexpr int kUnits = 4;

// Dv[h, r] = sum_c dO[r, h, c] * O[r, h, c] in fp32, and dQacc[h, r, :] = 0.
template <int D>
__global__ void __launch_bounds__(256) bwd_preprocess_kernel(const BwdArgs a) {
  constexpr int E = D / 32;  // bf16 elements per lane: 4 (8 bytes) or 2 (4 bytes)
  using V = typename std::conditional<E == 4, uint2, uint32_t>::type;
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

// dQ[r, h, :] = bf16(scale * dQacc[h, r, :]).
template <int D>
__global__ void __launch_bounds__(256) bwd_convert_kernel(const BwdArgs a) {
  constexpr int E = D / 32;  // fp32 elements per lane: 4 (16 bytes) or 2 (8 bytes)
  using F = typename std::conditional<E == 4, float4, float2>::type;
  const long long units = static_cast<long long>(a.total_q) * a.H;
  const long long u0 = ((static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * kUnits;
  const int lane = threadIdx.x & 31;
  if (u0 >= units) return;
  const float* acc = reinterpret_cast<const float*>(static_cast<const char*>(a.workspace) + a.dqacc_offset);
  F v[kUnits];
#pragma unroll
  for (int i = 0; i < kUnits; ++i) {
    const long long u = u0 + i;
    if (u < units) {
      const int row = static_cast<int>(u / a.H), h = static_cast<int>(u % a.H);
      v[i] = reinterpret_cast<const F*>(acc + (static_cast<size_t>(h) * a.tq_pad + row) * D)[lane];
    } else {
      v[i] = F{};
    }
  }
#pragma unroll
  for (int i = 0; i < kUnits; ++i) {
    const long long u = u0 + i;
    if (u >= units) break;
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.dq) + u * D;
    if constexpr (E == 4) {
      uint2 o;
      o.x = pack_bf16x2(v[i].x * a.scale, v[i].y * a.scale);
      o.y = pack_bf16x2(v[i].z * a.scale, v[i].w * a.scale);
      reinterpret_cast<uint2*>(dst)[lane] = o;
    } else {
      reinterpret_cast<uint32_t*>(dst)[lane] = pack_bf16x2(v[i].x * a.scale, v[i].y * a.scale);
    }
  }
}

template <int D, bool CAUSAL, bool DET>
cudaError_t launch_main(const BwdArgs& a, const BwdMaps& m, cudaStream_t stream) {
  using L = BwdSmem<D>;
  auto kern = bwd_kernel<D, CAUSAL, DET>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  kern<<<a.grid, kThreads, L::kAlloc, stream>>>(m.q, m.k, m.v, m.dout, m.dk, m.dv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_preprocess(const BwdArgs& a, cudaStream_t stream) {
  const long long warps = (static_cast<long long>(a.total_q) * a.H + kUnits - 1) / kUnits;
  const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
  if (blocks == 0) return cudaSuccess;
  if (a.D == 64)
    bwd_preprocess_kernel<64><<<blocks, 256, 0, stream>>>(a);
  else
    bwd_preprocess_kernel<128><<<blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
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
  if (a.D == 64)
    bwd_convert_kernel<64><<<blocks, 256, 0, stream>>>(a);
  else
    bwd_convert_kernel<128><<<blocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace fa
