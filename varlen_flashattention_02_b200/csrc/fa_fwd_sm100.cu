// fa_fwd_sm100.cu -- forward varlen attention for sm_100a.
//
// One persistent CTA per SM takes (sequence, head, query-tile) items from the
// scheduler's longest-first list through a global counter. For each item it computes, for
// 128 query rows of one head of one sequence, exact attention over the
// sequence's keys with an online softmax:
//
//   S_j   = Q K_j^T                      tcgen05.mma, bf16 -> fp32 in TMEM
//   m'    = max(m, rowmax(S_j) * scale)  registers, one thread per row
//   P_j   = exp2(S_j*scale*log2e - m')   registers -> bf16 back into TMEM
//   O     = O * exp2(m - m') + P_j V_j   tcgen05.mma with P read from TMEM
//   out   = O / l,  lse = (m + log2 l) * ln2
//
// Pages: "FlashAttention-2 GPU work partitioning" ("Bloques pequeños,
// normalización global": the running statistics and partial output are
// rescaled so that the normalisation stays global; "Tres mejoras": fewer
// non-matmul operations, parallelism over the sequence, queries split across
// workers that share K and V); "Flash-Atención y Flash-Atención-2" (tiles of
// Q, K, V are moved from HBM to on-chip memory and only the output goes
// back; FlashAttention-2 splits Q, not K, across warps so no cross-warp
// reduction is needed); "Mecanismo cu_seqlens en FlashAttention" ("Lógica de
// cálculo de longitud", "Optimización de acceso a memoria": per-sequence
// offsets and lengths from the cumulative arrays).
//
// B200 design, differing from the pages' A100 kernels:
//  * persistent grid of one CTA per SM over a longest-first work list
//    instead of one thread block per (batch, head[, q-block]);
//  * warp specialisation instead of 4-8 symmetric warps: warp 0 issues the
//    Q and K TMA loads, warp 2 the V loads (separate rings, so K can run
//    ahead of V), one thread of warp 1 issues tcgen05 MMAs, warps 4-7 (128
//    threads, one per query row and TMEM lane) do the softmax and epilogue;
//  * accumulators live in tensor memory (S double-buffered so QK^T of tile
//    j+1 overlaps the softmax of tile j; P overwrites its own S columns as
//    bf16 and feeds the PV MMA directly from TMEM);
//  * O is rescaled only when a row maximum grows by more than 2^8 (the
//    stale maximum stays consistent with l, so the result is exact);
//  * masking is applied only on the last key tile of a sequence and on
//    tiles that cross the causal diagonal; tiles wholly above it are never
//    loaded.
#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {
namespace {

constexpr int BM = kFwdBM;
constexpr int BN = kFwdBN;
constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kChunkBytes = 128 * 128;  // one [128 rows x 64 bf16] swizzled chunk
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct FwdSmem {
  // K and V have rings of their own: a K stage is released as soon as QK^T
  // has read it, a V stage only after PV, so K runs further ahead.
  static constexpr int kKStages = (D == 64) ? 4 : 3;
  static constexpr int kVStages = (D == 64) ? 4 : 2;
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;  // Q, K or V tile
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;                 // K stage s at kK + s*tile
  static constexpr int kV = kK + kKStages * kTileBytes;      // V stage s at kV + s*tile
  static constexpr int kBar = kV + kVStages * kTileBytes;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static constexpr int kSCol = 0;               // S buffers at columns 0 and 128
  static constexpr int kOCol = 256;             // O accumulator
};

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t o_full[2], o_empty;
  uint64_t drain;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  ItemRing items;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block fits its reserved space");

struct Item {
  int b, h, t;
  SeqInfo s;
  int nk;
};

__device__ __forceinline__ Item get_item(const FwdArgs& a, const int2* pairs, int idx) {
  Item it;
  const int2 pr = pairs[idx / a.H];
  it.h = idx % a.H;
  it.b = pr.x;
  it.t = pr.y;
  it.s = seq_info(a.cu_q, a.cu_k, it.b);
  it.nk = fwd_num_k_tiles(it.t, it.s.lq, it.s.lk, a.causal != 0);
  return it;
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  using L = FwdSmem<D>;
  constexpr int NK = L::kKStages, NV = L::kVStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(smem + L::kBar);

  auto* hdr = reinterpret_cast<WsHeader*>(a.workspace);
  const int2* pairs = reinterpret_cast<const int2*>(static_cast<const char*>(a.workspace) + a.pairs_offset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], 4);
    }
    mbar_init(&bars.o_full[0], 1);
    mbar_init(&bars.o_full[1], 1);
    mbar_init(&bars.o_empty, 4);
    mbar_init(&bars.drain, 1);
    for (int i = 0; i < NK; ++i) {
      mbar_init(&bars.k_full[i], 1);
      mbar_init(&bars.k_empty[i], 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&bars.v_full[i], 1);
      mbar_init(&bars.v_empty[i], 1);
    }
    // Item consumers: V producer (1), MMA warp (1), softmax warps (4).
    item_ring_init(bars.items, 6);
    bars.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(&bars.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;

  const Abort ab{&bars.abort_flag, &hdr->status};
  const int n_items = (hdr->status == FA_OK) ? static_cast<int>(hdr->n_pairs) * a.H : 0;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ Q and K producer
    uint32_t kc = 0, nq = 0, ni = 0;
    for (;;) {
      int idx;
      if (!publish_item(bars.items, ni, &hdr->work_counter, n_items, idx, ab)) goto kproducer_done;
      if (idx < 0) break;
      const Item it = get_item(a, pairs, idx);
      if (it.nk == 0) continue;
      if (nq > 0 && !wait_bar(&bars.q_empty, (nq - 1) & 1, ab)) goto kproducer_done;
      mbar_arrive_expect_tx(&bars.q_full, L::kTileBytes);
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_2d(&tm_q, &bars.q_full, smem + L::kQ + c * kChunkBytes, it.h * D + c * 64, it.s.q0 + it.t * BM);
      ++nq;
      for (int j = 0; j < it.nk; ++j, ++kc) {
        const int st = kc % NK;
        const uint32_t use = kc / NK;
        if (use > 0 && !wait_bar(&bars.k_empty[st], (use - 1) & 1, ab)) goto kproducer_done;
        mbar_arrive_expect_tx(&bars.k_full[st], L::kTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_2d(&tm_k, &bars.k_full[st], smem + L::kK + st * L::kTileBytes + c * kChunkBytes,
                      it.h * D + c * 64, it.s.k0 + j * BN);
      }
    }
  kproducer_done:
    // Never leave TMA writes in flight into shared memory we are about to
    // give up: wait (bounded) for the last loads issued.
    if (nq > 0) wait_bar_final(&bars.q_full, (nq - 1) & 1, ab);
    for (uint32_t i = (kc > NK ? kc - NK : 0); i < kc; ++i) wait_bar_final(&bars.k_full[i % NK], (i / NK) & 1, ab);
  } else if (warp == 2 && lane == 0) {
    // ------------------------------------------------------------ V producer
    uint32_t vc = 0, ni = 0;
    for (;;) {
      int slot;
      const int idx = consume_item<false>(bars.items, ni, slot, ab);
      if (idx < 0) break;
      mbar_arrive(&bars.items.empty[slot]);
      const Item it = get_item(a, pairs, idx);
      for (int j = 0; j < it.nk; ++j, ++vc) {
        const int st = vc % NV;
        const uint32_t use = vc / NV;
        if (use > 0 && !wait_bar(&bars.v_empty[st], (use - 1) & 1, ab)) goto vproducer_done;
        mbar_arrive_expect_tx(&bars.v_full[st], L::kTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_2d(&tm_v, &bars.v_full[st], smem + L::kV + st * L::kTileBytes + c * kChunkBytes,
                      it.h * D + c * 64, it.s.k0 + j * BN);
      }
    }
  vproducer_done:
    for (uint32_t i = (vc > NV ? vc - NV : 0); i < vc; ++i) wait_bar_final(&bars.v_full[i % NV], (i / NV) & 1, ab);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop converged (all values warp-uniform);
    // one elected lane issues each group of MMAs and the commits. Shared
    // memory descriptors are built once and advanced by constant offsets.
    constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, false, false);
    constexpr uint32_t kIdescO = idesc_bf16_f32(BM, D, false, true);
    const uint64_t q_desc = smem_desc_sw128(smem_u32(smem + L::kQ), 16, 1024);
    const uint64_t k_desc0 = smem_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
    const uint64_t v_desc0 = smem_desc_sw128(smem_u32(smem + L::kV), kChunkBytes, 1024);
    uint32_t kv = 0, g = 0, nq = 0, ni = 0;
    for (;;) {
      int slot;
      const int idx = consume_item<true>(bars.items, ni, slot, ab);
      if (idx < 0) break;
      if (elect_one()) mbar_arrive(&bars.items.empty[slot]);
      __syncwarp();
      const Item it = get_item(a, pairs, idx);
      if (it.nk == 0) continue;
      if (!wait_bar_warp(&bars.q_full, nq & 1, ab)) goto mma_done;
      tc_fence_after();
      for (int j = 0; j <= it.nk; ++j) {
        if (j < it.nk) {
          // S_j = Q K_j^T into S buffer (g + j) & 1.
          const uint32_t kvj = kv + j;
          const int st = kvj % NK;
          if (!wait_bar_warp(&bars.k_full[st], (kvj / NK) & 1, ab)) goto mma_done;
          tc_fence_after();
          const uint64_t k_desc = k_desc0 + static_cast<uint64_t>((st * L::kTileBytes) >> 4);
          const uint32_t d_s = tmem + L::kSCol + ((g + j) & 1) * BN;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
              mma_ss(d_s, q_desc + off, k_desc + off, kIdescS, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bars.s_full[(g + j) & 1]);
            mma_commit(&bars.k_empty[st]);
            if (j == it.nk - 1) mma_commit(&bars.q_empty);
          }
          __syncwarp();
        }
        if (j > 0) {
          // O (+)= P_{j-1} V_{j-1}, P read from TMEM.
          const int jj = j - 1;
          const uint32_t gj = g + jj, kvj = kv + jj;
          const int st = kvj % NV;
          if (!wait_bar_warp(&bars.p_full[gj & 1], (gj >> 1) & 1, ab)) goto mma_done;
          if (jj == 0 && nq > 0 && !wait_bar_warp(&bars.o_empty, (nq - 1) & 1, ab)) goto mma_done;
          if (!wait_bar_warp(&bars.v_full[st], (kvj / NV) & 1, ab)) goto mma_done;
          tc_fence_after();
          const uint64_t v_desc = v_desc0 + static_cast<uint64_t>((st * L::kTileBytes) >> 4);
          const uint32_t a_p = tmem + L::kSCol + (gj & 1) * BN;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              mma_ts(tmem + L::kOCol, a_p + kk * 8, v_desc + static_cast<uint64_t>((kk * 2048) >> 4), kIdescO,
                     (jj > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&bars.v_empty[st]);
            mma_commit(&bars.o_full[gj & 1]);
          }
          __syncwarp();
        }
      }
      kv += it.nk;
      g += it.nk;
      ++nq;
    }
  mma_done:
    // Make sure every MMA this warp issued has finished before TMEM is freed.
    if (elect_one()) mma_commit(&bars.drain);
    __syncwarp();
    wait_bar_final(&bars.drain, 0, ab);
  } else if (warp >= kSoftmaxWarp0) {
    // ------------------------------------------------------------ softmax
    const int row = threadIdx.x - kSoftmaxWarp0 * 32;  // query row in tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    uint32_t g = 0, nq = 0, ni = 0;
    for (;;) {
      int slot;
      const int idx = consume_item<true>(bars.items, ni, slot, ab);
      if (idx < 0) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.items.empty[slot]);
      const Item it = get_item(a, pairs, idx);
      const int r = it.t * BM + row;  // row within the sequence
      const bool row_ok = r < it.s.lq;
      const size_t orow = (static_cast<size_t>(it.s.q0) + r) * a.H + it.h;
      if (it.nk == 0) {
        if (row_ok) {
          uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow * D);
#pragma unroll
          for (int c = 0; c < D / 8; ++c) o[c] = make_uint4(0, 0, 0, 0);
          a.lse[static_cast<size_t>(it.h) * a.total_q + it.s.q0 + r] = -INFINITY;
        }
        continue;
      }
      float m_used = -INFINITY, l = 0.f;
      const int diag = it.s.lk - it.s.lq;  // key j visible from row i iff j <= i + diag
      for (int j = 0; j < it.nk; ++j, ++g) {
        const uint32_t buf = g & 1;
        if (!wait_bar_warp(&bars.s_full[buf], (g >> 1) & 1, ab)) goto softmax_done;
        tc_fence_after();
        uint32_t sr[BN];
        const uint32_t t_s = tmem + lane_base + L::kSCol + buf * BN;
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(t_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_wait_ld();
        float* s = reinterpret_cast<float*>(sr);
        const int key0 = j * BN;
        const bool need_mask = (key0 + BN > it.s.lk) || (CAUSAL && key0 + BN - 1 > it.t * BM + diag);
        if (need_mask) {
          int lim = it.s.lk - key0;
          if (CAUSAL) lim = min(lim, r + diag + 1 - key0);
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= lim) s[c] = -INFINITY;
        }
        // Row maximum: four independent chains of three-input maxima.
        float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
        for (int c = 4; c + 8 <= BN; c += 8) {
          m0 = fmax3(m0, s[c], s[c + 1]);
          m1 = fmax3(m1, s[c + 2], s[c + 3]);
          m2 = fmax3(m2, s[c + 4], s[c + 5]);
          m3 = fmax3(m3, s[c + 6], s[c + 7]);
        }
        m0 = fmax3(m0, s[BN - 4], s[BN - 3]);
        m1 = fmax3(m1, s[BN - 2], s[BN - 1]);
        const float mx = fmax3(m0, m1, fmaxf(m2, m3));
        const float m_new = fmaxf(m_used, mx * a.scale_log2);
        float alpha = 1.f;
        if (m_new > m_used + kRescaleThreshold) {
          alpha = ex2_approx(m_used - m_new);  // 0 when m_used = -inf
          l *= alpha;
          m_used = m_new;
        }
        if (__any_sync(0xffffffffu, j > 0 && alpha != 1.f)) {
          // O may be rescaled only once the previous PV (global index g-1)
          // has completed. PV completions alternate between two barriers, so
          // the phase waited for is unambiguous: S_g done implies PV_{g-2}
          // done, and PV_{g+1} cannot start before this tile's P exists.
          if (!wait_bar_warp(&bars.o_full[(g - 1) & 1], ((g - 1) >> 1) & 1, ab)) goto softmax_done;
          tc_fence_after();
          const uint32_t t_o = tmem + lane_base + L::kOCol;
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(t_o + c * 32, o);
          }
          tmem_wait_st();
        }
        const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
        // p = exp2(s * scale * log2e - m): pairs of columns share one packed
        // FMA and one packed add into the partial row sums.
        const uint64_t sc2 = f2_make(a.scale_log2, a.scale_log2);
        const uint64_t nm2 = f2_make(-m_ref, -m_ref);
        uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[BN / 2];
#pragma unroll
        for (int c = 0; c < BN; c += 2) {
          float x0, x1;
          f2_split(f2_fma(f2_make(s[c], s[c + 1]), sc2, nm2), x0, x1);
          const float p0 = ex2_approx(x0);
          const float p1 = ex2_approx(x1);
          ls2[(c >> 1) & 3] = f2_add(ls2[(c >> 1) & 3], f2_make(p0, p1));
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
        float ls4[4];
        {
          float a0, a1, b0, b1;
          f2_split(f2_add(ls2[0], ls2[1]), a0, a1);
          f2_split(f2_add(ls2[2], ls2[3]), b0, b1);
          ls4[0] = a0;
          ls4[1] = a1;
          ls4[2] = b0;
          ls4[3] = b1;
        }
        l += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
        // P (bf16, two per column) overwrites the first BN/2 columns of S.
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) tmem_st32(t_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[c * 32]));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[buf]);
      }
      // Epilogue: wait for the last PV (global index g-1), normalise, store.
      if (!wait_bar_warp(&bars.o_full[(g - 1) & 1], ((g - 1) >> 1) & 1, ab)) goto softmax_done;
      tc_fence_after();
      {
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        const uint32_t t_o = tmem + lane_base + L::kOCol;
        uint4* o_g = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow * D);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + c * 32, o);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint4 w;
              w.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
              w.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
              w.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
              w.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
              o_g[c * 4 + e] = w;
            }
          }
        }
        if (row_ok)
          a.lse[static_cast<size_t>(it.h) * a.total_q + it.s.q0 + r] =
              (l > 0.f) ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.o_empty);
      ++nq;
    }
  softmax_done:;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool CAUSAL>
cudaError_t launch_one(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       cudaStream_t stream) {
  using L = FwdSmem<D>;
  auto kern = fwd_kernel<D, CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  kern<<<a.grid, kThreads, L::kAlloc, stream>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       cudaStream_t stream) {
  if (a.D == 64) return a.causal ? launch_one<64, true>(a, tq, tk, tv, stream) : launch_one<64, false>(a, tq, tk, tv, stream);
  return a.causal ? launch_one<128, true>(a, tq, tk, tv, stream) : launch_one<128, false>(a, tq, tk, tv, stream);
}

}  // namespace fa
