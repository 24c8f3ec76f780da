// fa_bwd_d256_sm100.cu -- backward varlen attention for head_dim 256 (sm_100a).
//
// The page "Flash-Atención y Flash-Atención-2" (FlashAttention-2 section)
// extends the head dimension to 256. The gradients are those of the main
// backward (fa_bwd_sm100.cu), the chain rule of softmax attention with the
// probabilities recomputed from the saved logsumexp:
//
//   S^T = K_j Q_i^T,  P^T = exp2(S^T*scale*log2e - lse_i*log2e),
//   dP^T = V_j dO_i^T, dS^T = P^T * (dP^T - Dv_i),
//   dV_j = sum_i P^T dO_i,  dK_j = scale * sum_i dS^T Q_i,
//   dQ_i = scale * sum_j (K_j^T dS^T)^T   (fp32 bulk reductions, converted after).
//
// At d = 256 one CTA cannot hold both accumulators of a 128-key tile: dK and
// dV take 256 TMEM columns each, the whole of tensor memory, and K, V and a
// full-width Q/dO tile do not fit shared memory beside each other. The work
// is therefore split in two passes over the same (sequence, key/value head,
// key tile) work list, each of which fits on chip:
//  * pass 1, dV: S^T, P^T and dV += P^T dO over 128-query steps. TMEM: dV
//    (256 columns) and two S^T buffers of 128, so the next step's S^T runs
//    while this step's probabilities are computed. Shared memory: K and one
//    Q and one dO tile of 64 KB each.
//  * pass 2, dK and dQ: S^T, dP^T, P^T (registers), dS^T, dK += dS^T Q and
//    dQ^T = K^T dS^T over 64-query steps. TMEM: dK (256), S^T (64), dP^T
//    (64) and dQ^T as two 128-row halves of d (128). Shared memory: K, V
//    (64 KB each), one Q and one dO tile (32 KB each), dS^T (16 KB) and a
//    16 KB staging area for the dQ reductions.
// S^T is thus computed twice (six matrix products instead of five). dK/dV
// rows go to global memory straight from TMEM.
#include <type_traits>

#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {
namespace {

constexpr int D = 256;
constexpr int BN = kBwdBN;  // keys per item (128)
constexpr int kChunks = D / 64;
constexpr int kKChunk = BN * 128;  // [128 rows x 64 bf16] swizzled chunk
constexpr int kKTile = kChunks * kKChunk;  // 64 KB
constexpr uint32_t kTmemCols = 512;

// An item is (sequence, key/value head hk, key tile j); its steps visit the
// query tiles of `bm` rows that see the key tile, for each query head of the
// group: step s is query head h0 + s / nt, tile i0 + s % nt.
struct Item {
  int b, hk, j;
  SeqInfo s;
  int i0, nt, h0, n;
};

// Work order, as in the head_dim 64/128 backward: outside the deterministic
// mode the items are taken by cost class (longest class first, the work
// list's class_end) and head by head within a class, so that concurrent
// items mostly share a head whose Q/dO tiles and dQ accumulator rows stay in
// L2; the deterministic mode takes pair idx / Hk of head idx % Hk.
__device__ __forceinline__ Item get_item(const BwdArgs& a, const int2* pairs, int idx, int bm, int n_pairs,
                                         const uint32_t (&class_end)[kCostClasses]) {
  Item it;
  int pair = idx / a.Hk, hk = idx % a.Hk;
  if (!a.deterministic) {
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
  bwd_q_tiles(it.j, it.s.lq, it.s.lk, a.causal != 0, &it.i0, &e, bm);
  it.nt = e - it.i0;
  it.n = it.nt * a.group;
  return it;
}

struct Step {
  int h, t;
};
__device__ __forceinline__ Step item_step(const Item& it, int s) {
  const int r = s / it.nt;
  return Step{it.h0 + r, it.i0 + s - r * it.nt};
}

__device__ __forceinline__ uint4 pack8_bf16(const uint32_t* y, float scale) {
  uint4 w;
  w.x = pack_bf16x2(__uint_as_float(y[0]) * scale, __uint_as_float(y[1]) * scale);
  w.y = pack_bf16x2(__uint_as_float(y[2]) * scale, __uint_as_float(y[3]) * scale);
  w.z = pack_bf16x2(__uint_as_float(y[4]) * scale, __uint_as_float(y[5]) * scale);
  w.w = pack_bf16x2(__uint_as_float(y[6]) * scale, __uint_as_float(y[7]) * scale);
  return w;
}

// One row (TMEM lane) of a 256-column fp32 accumulator, times scale, as bf16
// to global memory, 32 columns at a time.
__device__ __forceinline__ void acc_row_to_global(uint32_t taddr, __nv_bfloat16* dst, float scale, bool store) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t x[32];
    tmem_ld32(taddr + c * 32, x);
    tmem_wait_ld();
    if (store) {
      uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
      for (int u = 0; u < 4; ++u) d4[u] = pack8_bf16(x + 8 * u, scale);
    }
  }
}

// Deterministic mode: wait for this query tile's turn (bounded).
__device__ __forceinline__ bool wait_turn(const uint32_t* cnt, uint32_t j, const Abort& ab) {
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

// ======================================================================
// Pass 1: dV. 256 threads: warp 0 lane 0 loads K and Q and hands out items,
// warp 1 issues MMAs, warp 2 lane 0 loads dO, warp 3 stages the logsumexp
// rows, warps 4-7 (one thread per key row = TMEM lane) compute P^T and write
// dV out at the end of each item.
namespace dv {
constexpr int BM = 128;  // queries per step
constexpr int kThreads = 256;
constexpr int kK = 0, kQ = kKTile, kDo = 2 * kKTile;
constexpr int kLd = 3 * kKTile;            // 2 slots x 128 fp32 (-lse * log2 e)
constexpr int kBar = kLd + 2 * BM * 4;
constexpr int kBytes = kBar + 512;
static_assert(kBytes <= 232448, "pass 1 fits shared memory");
constexpr int kColDV = 0, kColS = 256;     // S^T buffers at 256 and 384; P^T over their first 64 columns

struct Bars {
  uint64_t kv_full, kv_empty, q_full, q_empty, do_full, do_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t ld_full[2], ld_empty[2];
  uint64_t dv_full, dv_free, drain;
  ItemRing items;
  Item item_data[kItemSlots];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barriers fit");

template <bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_do, const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Bars& bars = *reinterpret_cast<Bars*>(smem + kBar);
  auto* hdr = reinterpret_cast<WsHeader*>(a.workspace);
  uint32_t* counter = &hdr->work_counter;
  const int2* pairs = reinterpret_cast<const int2*>(static_cast<const char*>(a.workspace) + a.pairs_offset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if ((smem_u32(smem) & 1023u) != 0) {  // swizzled tiles need a 1024-byte-aligned base
    griddep_wait();
    if (threadIdx.x == 0) atomicCAS(&hdr->status, 0u, static_cast<uint32_t>(FA_ERR_CUDA));
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(&bars.kv_full, 1);
    mbar_init(&bars.kv_empty, 1);
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    mbar_init(&bars.do_full, 1);
    mbar_init(&bars.do_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], 4);
      mbar_init(&bars.ld_full[i], 1);
      mbar_init(&bars.ld_empty[i], 4);
    }
    mbar_init(&bars.dv_full, 1);
    mbar_init(&bars.dv_free, 4);
    mbar_init(&bars.drain, 1);
    // Item consumers: MMA warp, dO loader, row loader, P warps (4).
    item_ring_init(bars.items, 7);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_do);
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
  const int n_items = (hdr->status == FA_OK) ? static_cast<int>(hdr->n_pairs) * a.Hk : 0;

  if (warp == 0) {
    if (lane == 0) {
      // K once per item, then Q of each step once the previous step's S^T
      // has read the single Q buffer.
      uint32_t m = 0, p = 0, ni = 0;
      const int n_pairs = static_cast<int>(hdr->n_pairs);
      uint32_t class_end[kCostClasses];
#pragma unroll
      for (int k = 0; k < kCostClasses; ++k) class_end[k] = hdr->class_end[k];
      for (;;) {
        int idx;
        Item it;
        auto decode = [&](int slot, int v) {
          it = get_item(a, pairs, v, BM, n_pairs, class_end);
          bars.item_data[slot] = it;
        };
        if (!publish_item_decoded(bars.items, ni, counter, n_items, idx, ab, decode)) goto k_done;
        if (idx < 0) break;
        if (it.n == 0) continue;
        const int krow = it.s.k0 + it.j * BN;
        for (int s = 0; s < it.n; ++s, ++p) {
          if (p > 0 && !wait_bar(&bars.q_empty, (p - 1) & 1, ab)) goto k_done;
          const Step sp = item_step(it, s);
          mbar_arrive_expect_tx(&bars.q_full, kKTile);
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d(&tm_q, &bars.q_full, smem + kQ + c * kKChunk, sp.h * D + c * 64, it.s.q0 + sp.t * BM);
          if (s == 0) {
            if (m > 0 && !wait_bar(&bars.kv_empty, (m - 1) & 1, ab)) {
              ++p;
              goto k_done;
            }
            mbar_arrive_expect_tx(&bars.kv_full, kKTile);
            for (int c = 0; c < kChunks; ++c)
              tma_load_2d(&tm_k, &bars.kv_full, smem + kK + c * kKChunk, it.hk * D + c * 64, krow);
            ++m;
          }
        }
      }
    k_done:
      if (m > 0) wait_bar_final(&bars.kv_full, (m - 1) & 1, ab);
      if (p > 0) wait_bar_final(&bars.q_full, (p - 1) & 1, ab);
    }
  } else if (warp == 1) {
    // Per step p: S^T(p) into buffer p % 2, then dV += P^T(p-1) dO(p-1) (the
    // previous step's probabilities), so S^T(p) overlaps P^T(p-1).
    constexpr uint32_t kIdS = idesc_bf16_f32(BN, BM, false, false);  // 128 x 128, K = 256
    constexpr uint32_t kIdV = idesc_bf16_f32(BN, D, false, true);    // 128 x 256, K = 128 queries
    const uint64_t k_kmaj = smem_desc_sw128(smem_u32(smem + kK), 16, 1024);
    const uint64_t q_kmaj = smem_desc_sw128(smem_u32(smem + kQ), 16, 1024);
    const uint64_t do_mn = smem_desc_sw128(smem_u32(smem + kDo), kKChunk, 1024);
    uint32_t m = 0, p = 0, ni = 0;
    auto issue_dv = [&](uint32_t pp, bool first) -> bool {
      const int b = pp & 1;
      if (!wait_bar_warp(&bars.p_full[b], (pp >> 1) & 1, ab)) return false;
      if (!wait_bar_warp(&bars.do_full, pp & 1, ab)) return false;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ts(tmem + kColDV, tmem + kColS + b * 128 + kk * 8, opaque_u64(do_mn) + ((kk * 2048) >> 4), kIdV,
                 (!first || kk > 0) ? 1u : 0u);
        mma_commit(&bars.do_empty);
      }
      __syncwarp();
      return true;
    };
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
      for (int s = 0; s < it.n; ++s, ++p) {
        if (!wait_bar_warp(&bars.q_full, p & 1, ab)) goto mma_done;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t o = ((kk >> 2) * kKChunk + (kk & 3) * 32) >> 4;
            mma_ss(tmem + kColS + (p & 1) * 128, opaque_u64(k_kmaj) + o, opaque_u64(q_kmaj) + o, kIdS, kk > 0);
          }
          mma_commit(&bars.s_full[p & 1]);
          mma_commit(&bars.q_empty);
        }
        __syncwarp();
        if (s > 0 && !issue_dv(p - 1, s == 1)) goto mma_done;
        if (s == 0 && m > 0 && !wait_bar_warp(&bars.dv_free, (m - 1) & 1, ab)) goto mma_done;
      }
      if (!issue_dv(p - 1, it.n == 1)) goto mma_done;
      if (elect_one()) {
        mma_commit(&bars.dv_full);
        mma_commit(&bars.kv_empty);
      }
      __syncwarp();
      ++m;
    }
  mma_done:
    if (elect_one()) mma_commit(&bars.drain);
    __syncwarp();
    wait_bar_final(&bars.drain, 0, ab);
  } else if (warp == 2) {
    if (lane == 0) {
      // dO of each step, once the previous step's dV has read the buffer.
      uint32_t p = 0, ni = 0;
      for (;;) {
        int slot;
        const int idx = consume_item<false>(bars.items, ni, slot, ab);
        if (idx < 0) break;
        const Item it = bars.item_data[slot];
        mbar_arrive(&bars.items.empty[slot]);
        for (int s = 0; s < it.n; ++s, ++p) {
          if (p > 0 && !wait_bar(&bars.do_empty, (p - 1) & 1, ab)) goto do_done;
          const Step sp = item_step(it, s);
          mbar_arrive_expect_tx(&bars.do_full, kKTile);
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d(&tm_do, &bars.do_full, smem + kDo + c * kKChunk, sp.h * D + c * 64, it.s.q0 + sp.t * BM);
        }
      }
    do_done:
      if (p > 0) wait_bar_final(&bars.do_full, (p - 1) & 1, ab);
    }
  } else if (warp == 3) {
    // -lse * log2(e) of the step's 128 query rows, four per thread.
    uint32_t p = 0, ni = 0;
    for (;;) {
      int islot;
      const int idx = consume_item<true>(bars.items, ni, islot, ab);
      if (idx < 0) break;
      const Item it = bars.item_data[islot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.items.empty[islot]);
      for (int s = 0; s < it.n; ++s, ++p) {
        const int slot = p & 1;
        if (p >= 2 && !wait_bar_warp(&bars.ld_empty[slot], ((p >> 1) - 1) & 1, ab)) goto ld_done;
        const Step sp = item_step(it, s);
        float* ld = reinterpret_cast<float*>(smem + kLd) + slot * BM;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = lane + 32 * u;
          const int qi = sp.t * BM + r;
          float v = -INFINITY;
          if (qi < it.s.lq) {
            const float l = __ldg(a.lse + static_cast<size_t>(sp.h) * a.total_q + it.s.q0 + qi);
            if (l != -INFINITY) v = -l * 1.4426950408889634f;
          }
          ld[r] = v;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.ld_full[slot]);
      }
    }
  ld_done:;
  } else {
    // P^T (warps 4-7, thread = key row = TMEM lane) and the dV epilogue.
    const int kr = threadIdx.x - 128;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t p = 0, m = 0, ni = 0;
    for (;;) {
      int islot;
      const int idx = consume_item<true>(bars.items, ni, islot, ab);
      if (idx < 0) break;
      const Item it = bars.item_data[islot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.items.empty[islot]);
      const int kg = it.j * BN + kr;
      const bool key_ok = kg < it.s.lk;
      const int diag = it.s.lk - it.s.lq;
      const size_t krow = (static_cast<size_t>(it.s.k0) + kg) * a.Hk + it.hk;
      __nv_bfloat16* dv_row = static_cast<__nv_bfloat16*>(a.dv) + krow * D;
      if (it.n == 0) {
        if (key_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dv_row);
#pragma unroll 4
          for (int c = 0; c < D / 8; ++c) d4[c] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      const uint64_t sc2 = f2_make(a.scale_log2, a.scale_log2);
      for (int s = 0; s < it.n; ++s, ++p) {
        const int b = p & 1;
        if (!wait_bar_warp(&bars.s_full[b], (p >> 1) & 1, ab)) goto p_done;
        if (!wait_bar_warp(&bars.ld_full[b], (p >> 1) & 1, ab)) goto p_done;
        tc_fence_after();
        const float* ld = reinterpret_cast<const float*>(smem + kLd) + b * BM;
        const uint32_t t_s = tmem + lane_base + kColS + b * 128;
        int e_min = CAUSAL ? kg - diag - item_step(it, s).t * BM : 0;
        if (!key_ok) e_min = BM;
#pragma unroll 1
        for (int c = 0; c < BM / 32; ++c) {
          uint32_t sv[32], pk[16];
          tmem_ld32(t_s + c * 32, sv);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int q = c * 32 + e;
            float x0, x1;
            f2_split(f2_fma(f2_make(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2,
                            *reinterpret_cast<const uint64_t*>(ld + q)),
                     x0, x1);
            float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            if (q < e_min) p0 = 0.f;
            if (q + 1 < e_min) p1 = 0.f;
            pk[e / 2] = pack_bf16x2(p0, p1);
          }
          // P^T columns 16c .. 16c+15 lie in columns already read.
          tmem_st16(t_s + c * 16, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars.p_full[b]);
          mbar_arrive(&bars.ld_empty[b]);
        }
      }
      // dV of the key tile: read out of TMEM (then released) and stored.
      if (!wait_bar_warp(&bars.dv_full, m & 1, ab)) goto p_done;
      tc_fence_after();
      acc_row_to_global(tmem + lane_base + kColDV, dv_row, 1.f, key_ok);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.dv_free);
      ++m;
    }
  p_done:;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}
}  // namespace dv

// ======================================================================
// Pass 2: dK and dQ. 384 threads: warp 0 lane 0 loads K, V, Q and dO and
// hands out items, warp 1 issues MMAs, warps 2-3 stage logsumexp and Dv
// rows, warps 4-7 (thread = key row) compute P^T and dS^T, warps 8-11 drain
// dQ^T into bulk fp32 reductions and write dK out at the end of each item.
namespace dkq {
constexpr int BM = 64;  // queries per step
constexpr int kThreads = 384;
constexpr int kQChunk = BM * 128;           // [64 rows x 64 bf16]
constexpr int kQTile = kChunks * kQChunk;   // 32 KB
constexpr int kK = 0, kV = kKTile, kQ = 2 * kKTile, kDo = kQ + kQTile;
constexpr int kDs = kDo + kQTile;           // dS^T [128 keys x 64 queries] bf16, 16 KB
constexpr int kStage = kDs + BN * BM * 2;   // dQ staging: 16 queries x 256 fp32 = 16 KB
constexpr int kStageRows = 16;
constexpr int kLd = kStage + kStageRows * D * 4;  // 2 slots x (lse[64], dv[64]) fp32
constexpr int kBar = kLd + 2 * 2 * BM * 4;
constexpr int kBytes = kBar + 512;
static_assert(kBytes <= 232448, "pass 2 fits shared memory");
constexpr int kColDK = 0, kColS = 256, kColDP = 320, kColDQ = 384;  // dQ^T half h at kColDQ + 64h

struct Bars {
  uint64_t kv_full, kv_empty, q_full, q_empty, do_full, do_empty;
  uint64_t s_full, dp_full, ds_full, dq_full, dq_free;
  uint64_t ld_full[2], ld_empty[2];
  uint64_t dk_full, dk_free, drain;
  ItemRing items;
  Item item_data[kItemSlots];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barriers fit");

template <bool CAUSAL, bool DET>
__global__ void __launch_bounds__(kThreads, 1)
    kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
           const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do, const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Bars& bars = *reinterpret_cast<Bars*>(smem + kBar);
  auto* hdr = reinterpret_cast<WsHeader*>(a.workspace);
  uint32_t* counter = &hdr->work_counter2;
  const int2* pairs = reinterpret_cast<const int2*>(static_cast<const char*>(a.workspace) + a.pairs_offset);
  const float* dvec = reinterpret_cast<const float*>(static_cast<const char*>(a.workspace) + a.dvec_offset);
  float* dqacc = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + a.dqacc_offset);
  uint32_t* qcount = reinterpret_cast<uint32_t*>(static_cast<char*>(a.workspace) + a.qcount_offset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if ((smem_u32(smem) & 1023u) != 0) {
    griddep_wait();
    if (threadIdx.x == 0) atomicCAS(&hdr->status, 0u, static_cast<uint32_t>(FA_ERR_CUDA));
    return;
  }
  if (threadIdx.x == 0) {
    mbar_init(&bars.kv_full, 1);
    mbar_init(&bars.kv_empty, 1);
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    mbar_init(&bars.do_full, 1);
    mbar_init(&bars.do_empty, 1);
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.dp_full, 1);
    mbar_init(&bars.ds_full, 4);
    mbar_init(&bars.dq_full, 1);
    mbar_init(&bars.dq_free, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.ld_full[i], 2);
      mbar_init(&bars.ld_empty[i], 4);
    }
    mbar_init(&bars.dk_full, 1);
    mbar_init(&bars.dk_free, 4);
    mbar_init(&bars.drain, 1);
    // Item consumers: MMA warp, row loaders (2), P/dS warps (4), drain warps (4).
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
  const int n_items = (hdr->status == FA_OK) ? static_cast<int>(hdr->n_pairs) * a.Hk : 0;

  if (warp == 0) {
    if (lane == 0) {
      // Per item K and V; per step dO (free once the previous dP^T is done)
      // and then Q (free once the previous dK MMA is done).
      uint32_t m = 0, nq = 0, nd = 0, ni = 0;  // K/V, Q and dO loads issued
      const int n_pairs = static_cast<int>(hdr->n_pairs);
      uint32_t class_end[kCostClasses];
#pragma unroll
      for (int k = 0; k < kCostClasses; ++k) class_end[k] = hdr->class_end[k];
      for (;;) {
        int idx;
        Item it;
        auto decode = [&](int slot, int v) {
          it = get_item(a, pairs, v, BM, n_pairs, class_end);
          bars.item_data[slot] = it;
        };
        if (!publish_item_decoded(bars.items, ni, counter, n_items, idx, ab, decode)) goto loads_done;
        if (idx < 0) break;
        if (it.n == 0) continue;
        const int krow = it.s.k0 + it.j * BN;
        for (int s = 0; s < it.n; ++s) {
          const Step sp = item_step(it, s);
          const int qrow = it.s.q0 + sp.t * BM;
          if (nd > 0 && !wait_bar(&bars.do_empty, (nd - 1) & 1, ab)) goto loads_done;
          mbar_arrive_expect_tx(&bars.do_full, kQTile);
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d(&tm_do, &bars.do_full, smem + kDo + c * kQChunk, sp.h * D + c * 64, qrow);
          ++nd;
          if (s == 0) {
            if (m > 0 && !wait_bar(&bars.kv_empty, (m - 1) & 1, ab)) goto loads_done;
            mbar_arrive_expect_tx(&bars.kv_full, 2 * kKTile);
            for (int c = 0; c < kChunks; ++c) {
              tma_load_2d(&tm_k, &bars.kv_full, smem + kK + c * kKChunk, it.hk * D + c * 64, krow);
              tma_load_2d(&tm_v, &bars.kv_full, smem + kV + c * kKChunk, it.hk * D + c * 64, krow);
            }
            ++m;
          }
          if (nq > 0 && !wait_bar(&bars.q_empty, (nq - 1) & 1, ab)) goto loads_done;
          mbar_arrive_expect_tx(&bars.q_full, kQTile);
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d(&tm_q, &bars.q_full, smem + kQ + c * kQChunk, sp.h * D + c * 64, qrow);
          ++nq;
        }
      }
    loads_done:
      // Every load issued must land before shared memory is given up.
      if (nd > 0) wait_bar_final(&bars.do_full, (nd - 1) & 1, ab);
      if (nq > 0) wait_bar_final(&bars.q_full, (nq - 1) & 1, ab);
      if (m > 0) wait_bar_final(&bars.kv_full, (m - 1) & 1, ab);
    }
  } else if (warp == 1) {
    // Per step: S^T = K Q^T; dP^T = V dO^T; [dS^T written] dK += dS^T Q;
    // [dQ^T of the previous step read out] dQ^T = K^T dS^T (two 128-row
    // halves of d).
    constexpr uint32_t kIdS = idesc_bf16_f32(BN, BM, false, false);   // 128 x 64, K = 256
    constexpr uint32_t kIdK = idesc_bf16_f32(BN, D, false, true);     // 128 x 256, K = 64 queries
    constexpr uint32_t kIdQ = idesc_bf16_f32(128, BM, true, true);    // 128 (d half) x 64, K = 128 keys
    const uint64_t k_kmaj = smem_desc_sw128(smem_u32(smem + kK), 16, 1024);
    const uint64_t v_kmaj = smem_desc_sw128(smem_u32(smem + kV), 16, 1024);
    const uint64_t k_mn = smem_desc_sw128(smem_u32(smem + kK), kKChunk, 1024);
    const uint64_t q_kmaj = smem_desc_sw128(smem_u32(smem + kQ), 16, 1024);
    const uint64_t do_kmaj = smem_desc_sw128(smem_u32(smem + kDo), 16, 1024);
    const uint64_t q_mn = smem_desc_sw128(smem_u32(smem + kQ), kQChunk, 1024);
    const uint64_t ds_mn = smem_desc_sw128(smem_u32(smem + kDs), 0, 1024);
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
      for (int s = 0; s < it.n; ++s, ++p) {
        if (!wait_bar_warp(&bars.q_full, p & 1, ab)) goto mma_done;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ok = ((kk >> 2) * kKChunk + (kk & 3) * 32) >> 4;
            const uint64_t oq = ((kk >> 2) * kQChunk + (kk & 3) * 32) >> 4;
            mma_ss(tmem + kColS, opaque_u64(k_kmaj) + ok, opaque_u64(q_kmaj) + oq, kIdS, kk > 0);
          }
          mma_commit(&bars.s_full);
        }
        __syncwarp();
        if (!wait_bar_warp(&bars.do_full, p & 1, ab)) goto mma_done;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t ok = ((kk >> 2) * kKChunk + (kk & 3) * 32) >> 4;
            const uint64_t oq = ((kk >> 2) * kQChunk + (kk & 3) * 32) >> 4;
            mma_ss(tmem + kColDP, opaque_u64(v_kmaj) + ok, opaque_u64(do_kmaj) + oq, kIdS, kk > 0);
          }
          mma_commit(&bars.dp_full);
          mma_commit(&bars.do_empty);
        }
        __syncwarp();
        if (!wait_bar_warp(&bars.ds_full, p & 1, ab)) goto mma_done;
        if (s == 0 && m > 0 && !wait_bar_warp(&bars.dk_free, (m - 1) & 1, ab)) goto mma_done;
        tc_fence_after();
        if (elect_one()) {
          // dK += dS^T Q: dS^T bf16 in TMEM over the S^T columns (16 queries
          // = 8 columns per MMA), Q MN-major.
#pragma unroll
          for (int kk = 0; kk < BM / 16; ++kk)
            mma_ts(tmem + kColDK, tmem + kColS + kk * 8, opaque_u64(q_mn) + ((kk * 16 * 128) >> 4), kIdK,
                   (s > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars.q_empty);
        }
        __syncwarp();
        if (p > 0 && !wait_bar_warp(&bars.dq_free, (p - 1) & 1, ab)) goto mma_done;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              mma_ss(tmem + kColDQ + h * 64, opaque_u64(k_mn) + ((2 * h * kKChunk + kk * 2048) >> 4),
                     opaque_u64(ds_mn) + ((kk * 2048) >> 4), kIdQ, kk > 0);
          mma_commit(&bars.dq_full);
        }
        __syncwarp();
      }
      if (elect_one()) {
        mma_commit(&bars.dk_full);
        mma_commit(&bars.kv_empty);
      }
      __syncwarp();
      ++m;
    }
  mma_done:
    if (elect_one()) mma_commit(&bars.drain);
    __syncwarp();
    wait_bar_final(&bars.drain, 0, ab);
  } else if (warp < 4) {
    // -lse * log2(e) and Dv of the step's 64 query rows, one per thread.
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
        const int slot = p & 1;
        if (p >= 2 && !wait_bar_warp(&bars.ld_empty[slot], ((p >> 1) - 1) & 1, ab)) goto rows_done;
        const Step sp = item_step(it, s);
        const int qi = sp.t * BM + r;
        float nl = -INFINITY, dv = 0.f;
        if (qi < it.s.lq) {
          const size_t gq = static_cast<size_t>(it.s.q0) + qi;
          const float l = __ldg(a.lse + static_cast<size_t>(sp.h) * a.total_q + gq);
          if (l != -INFINITY) {
            nl = -l * 1.4426950408889634f;
            dv = __ldg(dvec + static_cast<size_t>(sp.h) * a.tq_pad + gq);
          }
        }
        float* ld = reinterpret_cast<float*>(smem + kLd) + slot * 2 * BM;
        ld[r] = nl;
        ld[BM + r] = dv;
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.ld_full[slot]);
      }
    }
  rows_done:;
  } else if (warp < 8) {
    // P^T (kept in registers as bf16 pairs) and dS^T = P^T (dP^T - Dv), to
    // TMEM (A operand of dK) and shared memory (B operand of dQ^T).
    const int kr = threadIdx.x - 128;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint8_t* ds_row = smem + kDs + kr * 128;
    uint32_t p = 0, ni = 0;
    for (;;) {
      int islot;
      const int idx = consume_item<true>(bars.items, ni, islot, ab);
      if (idx < 0) break;
      const Item it = bars.item_data[islot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.items.empty[islot]);
      const int kg = it.j * BN + kr;
      const bool key_ok = kg < it.s.lk;
      const int diag = it.s.lk - it.s.lq;
      const uint64_t sc2 = f2_make(a.scale_log2, a.scale_log2);
      for (int s = 0; s < it.n; ++s, ++p) {
        const int slot = p & 1;
        if (!wait_bar_warp(&bars.s_full, p & 1, ab)) goto pds_done;
        if (!wait_bar_warp(&bars.ld_full[slot], (p >> 1) & 1, ab)) goto pds_done;
        tc_fence_after();
        const float* ld = reinterpret_cast<const float*>(smem + kLd) + slot * 2 * BM;
        int e_min = CAUSAL ? kg - diag - item_step(it, s).t * BM : 0;
        if (!key_ok) e_min = BM;
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32];
          tmem_ld32(tmem + lane_base + kColS + c * 32, sv);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int q = c * 32 + e;
            float x0, x1;
            f2_split(f2_fma(f2_make(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2,
                            *reinterpret_cast<const uint64_t*>(ld + q)),
                     x0, x1);
            float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            if (q < e_min) p0 = 0.f;
            if (q + 1 < e_min) p1 = 0.f;
            pk[q / 2] = pack_bf16x2(p0, p1);
          }
        }
        if (!wait_bar_warp(&bars.dp_full, p & 1, ab)) goto pds_done;
        // The dQ^T MMAs of the previous step must have read dS^T from shared
        // memory before it is overwritten.
        if (p > 0 && !wait_bar_warp(&bars.dq_full, (p - 1) & 1, ab)) goto pds_done;
        tc_fence_after();
        const uint64_t* dv2 = reinterpret_cast<const uint64_t*>(ld + BM);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t dpv[32], dsk[16];
          tmem_ld32(tmem + lane_base + kColDP + c * 32, dpv);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int q = c * 32 + e;
            const uint32_t pp = pk[q / 2];
            float d0, d1;
            f2_split(f2_mul(f2_make(__uint_as_float(pp << 16), __uint_as_float(pp & 0xffff0000u)),
                            f2_sub(f2_make(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])), dv2[q / 2])),
                     d0, d1);
            dsk[e / 2] = pack_bf16x2(d0, d1);
          }
          // dS^T into TMEM columns 16c .. 16c+15 of the S^T block (already
          // read) and into shared memory row kr (128-byte swizzle).
          tmem_st16(tmem + lane_base + kColS + c * 16, dsk);
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
  pds_done:;
  } else {
    // dQ^T drain (thread = d within a half = TMEM lane) and the dK epilogue
    // (thread = key row).
    const int t = threadIdx.x - 256;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float* stage = reinterpret_cast<float*>(smem + kStage);
    uint32_t p = 0, m = 0, ni = 0;
    uint32_t* det_prev = nullptr;
    for (;;) {
      int islot;
      const int idx = consume_item<true>(bars.items, ni, islot, ab);
      if (!named_bar_and(1, 128, idx >= 0)) break;
      const Item it = bars.item_data[islot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.items.empty[islot]);
      const int kg = it.j * BN + t;
      const bool key_ok = kg < it.s.lk;
      __nv_bfloat16* dk_row =
          static_cast<__nv_bfloat16*>(a.dk) + ((static_cast<size_t>(it.s.k0) + kg) * a.Hk + it.hk) * D;
      if (it.n == 0) {
        if (key_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dk_row);
#pragma unroll 4
          for (int c = 0; c < D / 8; ++c) d4[c] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      for (int s = 0; s < it.n; ++s, ++p) {
        if (!named_bar_and(1, 128, wait_bar(&bars.dq_full, p & 1, ab))) goto drain_done;
        tc_fence_after();
        const Step sp = item_step(it, s);
        const size_t q0 = static_cast<size_t>(it.s.q0) + static_cast<size_t>(sp.t) * BM;
        uint32_t* cnt = qcount + static_cast<size_t>(sp.h) * a.tq_pad + q0;
        if (DET && t == 0) wait_turn(cnt, static_cast<uint32_t>(it.j), ab);
        // 16 query rows at a time: both d halves of each row, so that the
        // staged rows are one contiguous block of the head-major accumulator.
#pragma unroll 1
        for (int g = 0; g < BM / kStageRows; ++g) {
          uint32_t v0[16], v1[16];
          tmem_ld16(tmem + lane_base + kColDQ + g * 16, v0);
          tmem_ld16(tmem + lane_base + kColDQ + 64 + g * 16, v1);
          tmem_wait_ld();
          if (g == BM / kStageRows - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.dq_free);
          }
          if (t == 0) bulk_wait_group_read0();
          named_bar_sync(1, 128);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            stage[e * D + t] = __uint_as_float(v0[e]);
            stage[e * D + 128 + t] = __uint_as_float(v1[e]);
          }
          fence_proxy_async_smem();
          named_bar_sync(1, 128);
          if (t == 0 && !*ab.flag) {
            if (DET) fence_proxy_async_global();
            bulk_reduce_add_f32(dqacc + (static_cast<size_t>(sp.h) * a.tq_pad + q0 + g * kStageRows) * D, stage,
                                kStageRows * D * 4);
            bulk_commit_group();
          }
        }
        if (DET && t == 0 && !*ab.flag) {
          // Pass the previous step's turn on once its additions are done.
          if (det_prev) {
            bulk_wait_group4();
            fence_proxy_async_global();
            st_release_gpu(det_prev, static_cast<uint32_t>(it.j) + 1u);
          }
          det_prev = cnt;
        }
      }
      if (DET && t == 0 && det_prev) {
        bulk_wait_group0();
        fence_proxy_async_global();
        st_release_gpu(det_prev, static_cast<uint32_t>(it.j) + 1u);
        det_prev = nullptr;
      }
      if (!named_bar_and(1, 128, wait_bar(&bars.dk_full, m & 1, ab))) goto drain_done;
      tc_fence_after();
      acc_row_to_global(tmem + lane_base + kColDK, dk_row, a.scale, key_ok);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.dk_free);
      ++m;
    }
  drain_done:
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
}  // namespace dkq

template <class K>
cudaError_t prepare(K kern, int bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

cudaError_t launch_bwd_d256(const BwdArgs& a, const BwdMapsD256& m, cudaStream_t stream) {
  cudaError_t e;
  auto k1 = a.causal ? dv::kernel<true> : dv::kernel<false>;
  if ((e = prepare(k1, dv::kBytes)) != cudaSuccess) return e;
  if ((e = launch_kernel(k1, a.grid, dv::kThreads, dv::kBytes, stream, a.chained != 0, m.q128, m.k, m.do128, a)) !=
      cudaSuccess)
    return e;
  auto k2 = a.causal ? (a.deterministic ? dkq::kernel<true, true> : dkq::kernel<true, false>)
                     : (a.deterministic ? dkq::kernel<false, true> : dkq::kernel<false, false>);
  if ((e = prepare(k2, dkq::kBytes)) != cudaSuccess) return e;
  return launch_kernel(k2, a.grid, dkq::kThreads, dkq::kBytes, stream, a.chained != 0, m.q64, m.k, m.v, m.do64, a);
}

}  // namespace fa
