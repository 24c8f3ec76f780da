// fa_fwd_d256_sm100.cu -- forward varlen attention for head_dim 256 (sm_100a).
//
// The page "Flash-Atención y Flash-Atención-2" notes that FlashAttention-2
// extends the head dimension to 256. The computation is the same as the
// main forward (fa_fwd_sm100.cu): per (sequence, head, 128-row query tile),
// an online softmax over key tiles,
//
//   S_j = Q K_j^T,  m' = max(m, rowmax(S_j) * scale),  P_j = exp2(...),
//   O = O * exp2(m - m') + P_j V_j,  out = O / l,  lse = (m + log2 l) ln 2,
//
// only the tiling differs, because at d = 256 the output accumulator alone
// takes 256 of the 512 TMEM columns:
//  * one 128-row query tile per CTA (the work list has 128-row items);
//  * key tiles of 64 keys: S_j is 128 x 64 fp32 and is double-buffered in
//    TMEM (columns 0 and 64) so Q K_{j+1}^T overlaps the softmax of tile j;
//    O occupies columns 256-511; P overwrites its S columns as bf16;
//  * shared memory: Q 64 KB, K ring 3 x 32 KB, V ring 2 x 32 KB;
//  * PV is M = 128, N = 256: the widest MMA shape, the most work per issued
//    instruction;
//  * one warp issues Q and K loads (and hands out items), one V loads, one
//    MMAs; four warps (one thread per query row) run the softmax and the
//    epilogue.
// Masking, lazy rescaling, grouped heads and the key layouts (packed,
// cache slots, pages) are those of the main forward.
#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {
namespace {

constexpr int D = 256;
constexpr int BM = kFwdBM;  // query rows per item
constexpr int BN = 64;      // keys per tile
constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kChunks = D / 64;                    // 64-column chunks of a row
constexpr int kQChunkBytes = BM * 128;             // [128 rows x 64 bf16], 128-byte swizzle
constexpr int kKVChunkBytes = BN * 128;            // [64 rows x 64 bf16]
constexpr int kQBytes = kChunks * kQChunkBytes;    // 64 KB
constexpr int kKVBytes = kChunks * kKVChunkBytes;  // 32 KB per K or V tile
constexpr int kKStages = 3, kVStages = 2;
constexpr int kSmemQ = 0;
constexpr int kSmemK = kSmemQ + kQBytes;
constexpr int kSmemV = kSmemK + kKStages * kKVBytes;
constexpr int kSmemBar = kSmemV + kVStages * kKVBytes;
constexpr int kSmemBytes = kSmemBar + 512;
constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-byte alignment
static_assert(kSmemAlloc <= 232448, "layout fits 227 KB of shared memory");
constexpr uint32_t kTmemCols = 512;
constexpr int kSCol = 0;    // S buffers at columns 0 and BN
constexpr int kOCol = 256;  // O: D columns
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t s_full[2], p_full[2];
  uint64_t o_full[2], o_empty;
  uint64_t drain;
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  ItemRing items;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block fits its reserved space");

struct Item {
  int b, h, hk, t;  // t: 128-row query tile of the sequence
  SeqInfo s;
  int nk;           // key tiles (of BN) visible from the tile
};

__device__ __forceinline__ Item get_item(const FwdArgs& a, const int2* pairs, int idx) {
  Item it;
  const int2 pr = pairs[idx / a.H];
  it.h = idx % a.H;
  it.hk = it.h / a.group;
  it.b = pr.x;
  it.t = pr.y;
  it.s = seq_info(a.cu_q, a.keys, it.b);
  it.nk = fwd_k_tiles((it.t + 1) * BM, it.s.lq, it.s.lk, a.causal != 0, BN);
  return it;
}

template <bool CAUSAL>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_d256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(smem + kSmemBar);
  auto* hdr = reinterpret_cast<WsHeader*>(a.workspace);
  const int2* pairs = reinterpret_cast<const int2*>(static_cast<const char*>(a.workspace) + a.pairs_offset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], 4);
      mbar_init(&bars.o_full[i], 1);
    }
    mbar_init(&bars.o_empty, 4);
    mbar_init(&bars.drain, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bars.k_full[i], 1);
      mbar_init(&bars.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
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
  // Everything above is local to the CTA; the work list, the inputs and the
  // outputs are touched only after the work-list kernel has finished.
  griddep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  const Abort ab{&bars.abort_flag, &hdr->status, a.wait_ns};
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
      mbar_arrive_expect_tx(&bars.q_full, kQBytes);
      for (int c = 0; c < kChunks; ++c)
        tma_load_2d(&tm_q, &bars.q_full, smem + kSmemQ + c * kQChunkBytes, it.h * D + c * 64, it.s.q0 + it.t * BM);
      ++nq;
      for (int j = 0; j < it.nk; ++j, ++kc) {
        const int st = kc % kKStages;
        const uint32_t use = kc / kKStages;
        const int krow = key_tile_row(a.keys, it.b, it.s, j, BN);
        if (use > 0 && !wait_bar(&bars.k_empty[st], (use - 1) & 1, ab)) goto kproducer_done;
        mbar_arrive_expect_tx(&bars.k_full[st], kKVBytes);
        for (int c = 0; c < kChunks; ++c)
          tma_load_2d(&tm_k, &bars.k_full[st], smem + kSmemK + st * kKVBytes + c * kKVChunkBytes, it.hk * D + c * 64,
                      krow);
      }
    }
  kproducer_done:
    // Never leave TMA writes in flight into shared memory that is about to be
    // given up: wait (bounded) for the last loads issued.
    if (nq > 0) wait_bar_final(&bars.q_full, (nq - 1) & 1, ab);
    for (uint32_t i = (kc > kKStages ? kc - kKStages : 0); i < kc; ++i)
      wait_bar_final(&bars.k_full[i % kKStages], (i / kKStages) & 1, ab);
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
        const int st = vc % kVStages;
        const uint32_t use = vc / kVStages;
        const int vrow = key_tile_row(a.keys, it.b, it.s, j, BN);
        if (use > 0 && !wait_bar(&bars.v_empty[st], (use - 1) & 1, ab)) goto vproducer_done;
        mbar_arrive_expect_tx(&bars.v_full[st], kKVBytes);
        for (int c = 0; c < kChunks; ++c)
          tma_load_2d(&tm_v, &bars.v_full[st], smem + kSmemV + st * kKVBytes + c * kKVChunkBytes, it.hk * D + c * 64,
                      vrow);
      }
    }
  vproducer_done:
    for (uint32_t i = (vc > kVStages ? vc - kVStages : 0); i < vc; ++i)
      wait_bar_final(&bars.v_full[i % kVStages], (i / kVStages) & 1, ab);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop converged; one elected lane issues each
    // group of MMAs and the commits. Order per key tile: S_j = Q K_j^T (into
    // S buffer (g + j) & 1), then O (+)= P_{j-1} V_{j-1}; S_{j+1} overwrites
    // P_{j-1} only after that PV was issued, and MMAs execute in issue order.
    constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, false, false);  // 128 x 64, K-major A and B
    constexpr uint32_t kIdescO = idesc_bf16_f32(BM, D, false, true);    // 128 x 256, V MN-major
    const uint64_t q_desc = smem_desc_sw128(smem_u32(smem + kSmemQ), 16, 1024);
    const uint64_t k_desc0 = smem_desc_sw128(smem_u32(smem + kSmemK), 16, 1024);
    // V: N (= d) runs along the rows of a chunk; consecutive 64-column
    // chunks are kKVChunkBytes apart.
    const uint64_t v_desc0 = smem_desc_sw128(smem_u32(smem + kSmemV), kKVChunkBytes, 1024);
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
          const uint32_t kvj = kv + j;
          const int st = kvj % kKStages;
          if (!wait_bar_warp(&bars.k_full[st], (kvj / kKStages) & 1, ab)) goto mma_done;
          tc_fence_after();
          const uint64_t k_desc = opaque_u64(k_desc0) + static_cast<uint64_t>((st * kKVBytes) >> 4);
          const uint32_t d_s = tmem + kSCol + ((g + j) & 1) * BN;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t oq = static_cast<uint64_t>(((kk >> 2) * kQChunkBytes + (kk & 3) * 32) >> 4);
              const uint64_t ok = static_cast<uint64_t>(((kk >> 2) * kKVChunkBytes + (kk & 3) * 32) >> 4);
              mma_ss(d_s, q_desc + oq, k_desc + ok, kIdescS, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bars.s_full[(g + j) & 1]);
            mma_commit(&bars.k_empty[st]);
            if (j == it.nk - 1) mma_commit(&bars.q_empty);
          }
          __syncwarp();
        }
        if (j > 0) {
          const int jj = j - 1;
          const uint32_t gj = g + jj, kvj = kv + jj;
          const int st = kvj % kVStages;
          if (jj == 0 && nq > 0 && !wait_bar_warp(&bars.o_empty, (nq - 1) & 1, ab)) goto mma_done;
          if (!wait_bar_warp(&bars.v_full[st], (kvj / kVStages) & 1, ab)) goto mma_done;
          const uint64_t v_desc = opaque_u64(v_desc0) + static_cast<uint64_t>((st * kKVBytes) >> 4);
          const uint32_t a_p = tmem + kSCol + (gj & 1) * BN;
          if (!wait_bar_warp(&bars.p_full[gj & 1], (gj >> 1) & 1, ab)) goto mma_done;
          tc_fence_after();
          if (elect_one()) {
            // O (+)= P V: P (bf16, two per column) from TMEM, 16 keys per MMA.
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              mma_ts(tmem + kOCol, a_p + kk * 8, v_desc + static_cast<uint64_t>((kk * 2048) >> 4), kIdescO,
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
    // ------------------------------------------------------------ softmax and epilogue
    const int row = threadIdx.x - kSoftmaxWarp0 * 32;  // query row in tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_o = tmem + lane_base + kOCol;
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
      uint4* o_g = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow * D);
      float* lse_g = a.lse + static_cast<size_t>(it.h) * a.total_q + it.s.q0 + r;
      if (it.nk == 0) {
        if (row_ok) {
#pragma unroll 4
          for (int c = 0; c < D / 8; ++c) o_g[c] = make_uint4(0, 0, 0, 0);
          *lse_g = -INFINITY;
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
        const uint32_t t_s = tmem + lane_base + kSCol + buf * BN;
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
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_o + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(t_o + c * 32, o);
          }
        }
        const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
        // p = exp2(s * scale * log2e - m), pairs of columns in packed f32x2
        // arithmetic; P (bf16, two per column) overwrites the first BN/2
        // columns of S.
        const uint64_t sc2 = f2_make(a.scale_log2, a.scale_log2);
        const uint64_t nm2 = f2_make(-m_ref, -m_ref);
        uint64_t ls2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int hh = 0; hh < BN / 32; ++hh) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            float x0, x1;
            f2_split(f2_fma(f2_make(s[hh * 32 + c], s[hh * 32 + c + 1]), sc2, nm2), x0, x1);
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            ls2[(c >> 1) & 3] = f2_add(ls2[(c >> 1) & 3], f2_make(p0, p1));
            pk[c / 2] = pack_bf16x2(p0, p1);
          }
          tmem_st16(t_s + hh * 16, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.p_full[buf]);
        {
          float a0, a1, b0, b1;
          f2_split(f2_add(ls2[0], ls2[1]), a0, a1);
          f2_split(f2_add(ls2[2], ls2[3]), b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
      }
      // Epilogue: wait for the last PV (global index g-1), normalise, store.
      if (!wait_bar_warp(&bars.o_full[(g - 1) & 1], ((g - 1) >> 1) & 1, ab)) goto softmax_done;
      tc_fence_after();
      {
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
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
        if (row_ok) *lse_g = (l > 0.f) ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
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

template <bool CAUSAL>
cudaError_t launch_one(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       cudaStream_t stream) {
  auto kern = fwd_d256_kernel<CAUSAL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, a.grid, kThreads, kSmemAlloc, stream, a.chained != 0, tq, tk, tv, a);
}

}  // namespace

cudaError_t launch_fwd_d256(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            cudaStream_t stream) {
  if (a.D != D) return cudaErrorInvalidValue;
  return a.causal ? launch_one<true>(a, tq, tk, tv, stream) : launch_one<false>(a, tq, tk, tv, stream);
}

}  // namespace fa
