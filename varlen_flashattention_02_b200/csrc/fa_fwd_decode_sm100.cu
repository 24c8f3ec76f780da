// fa_fwd_decode_sm100.cu -- split-KV forward with grouped query heads
// packed into one tile (sm_100a), for decoding and other short-query calls.
//
// The page "FlashAttention-2 GPU work partitioning" ("Cómo documentar una
// diferencia técnica") separates prefill from token-by-token decoding, whose
// bottleneck differs: with one or a few query tokens per sequence a
// 128-row query tile is almost empty and there are too few (sequence,
// head) items to occupy 148 SMs, while the key/value cache has to be
// streamed from HBM. Two changes to the forward's work decomposition
// address that (the computation itself, exact attention with an online
// softmax, is the main forward's):
//  * the g query heads that share a key/value head ("Flash-Atención y
//    Flash-Atención-2", FlashAttention-2 section) and 128 / g consecutive
//    query tokens fill the 128 rows of one tile (row m = token m / g, head
//    m % g of the group): a 3-D TMA box (64 dims x g heads x 128/g tokens)
//    lands exactly these rows, and each K/V tile is read once for the whole
//    group;
//  * the key tiles of an item are split into `splits` ranges processed by
//    different CTAs; each writes its normalised partial output and its
//    logsumexp, and the combine kernel merges them:
//      lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) * out_s.
// Items come from the work list, or, when every sequence fits one query tile
// (decoding), straight from their index, each sequence then checked by the
// kernel itself. Roles: one warp loads Q and K (and hands out items), one
// loads V, one issues the MMAs, four (one thread per tile row) run the
// softmax and the epilogue; S is double-buffered in TMEM, O accumulates in
// TMEM.
#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {
namespace {

constexpr int BM = 128;  // tile rows
constexpr int BN = 128;  // keys per tile
constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kChunkBytes = 128 * 128;  // [128 rows x 64 bf16], 128-byte swizzle
constexpr uint32_t kTmemCols = 512;
constexpr int kSCol = 0;    // S buffers at columns 0 and 128
constexpr int kOCol = 256;  // O
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct DecSmem {
  static constexpr int kKStages = (D == 64) ? 4 : 3;
  static constexpr int kVStages = (D == 64) ? 4 : 2;
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kKStages * kTileBytes;
  static constexpr int kBar = kV + kVStages * kTileBytes;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
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
  int b, hk, t, split;  // t: tile of tq query tokens
  SeqInfo s;
  int j0, j1;           // key tiles [j0, j1) of this split
  bool bad;             // inline list: the sequence failed its checks (the item does nothing)
};

// Without a work list, the checks the work-list kernel makes on sequence b:
// its query rows lie inside [0, total_q) and number at most max_seqlen_q,
// and its keys lie inside their layout's bounds (packed: inside [0,
// total_k); cache slots: 0 <= leftpad <= seqlens <= cache_rows; pages: at
// most max_pages * page_size keys) and number at most max_seqlen_k.
template <int KL>
__device__ __forceinline__ bool seq_ok(const DecodeArgs& a, int b, const SeqInfo& s) {
  if (s.q0 < 0 || s.lq < 0 || s.lq > a.max_seqlen_q || s.q0 + s.lq > a.total_q) return false;
  if (s.lk < 0 || s.lk > a.max_seqlen_k) return false;
  if (KL == kKeysPaged) return s.lk <= a.keys.max_pages * a.keys.page_size;
  if (KL == kKeysSlots) {
    const int lp = a.keys.leftpad_k ? __ldg(a.keys.leftpad_k + b) : 0;
    return lp >= 0 && lp + s.lk <= a.keys.cache_rows;
  }
  return s.k0 >= 0 && s.k0 + s.lk <= a.total_k;
}

template <int KL>
__device__ __forceinline__ Item get_item(const DecodeArgs& a, const int2* pairs, int idx) {
  Item it;
  it.split = idx % a.splits;
  const int rest = idx / a.splits;
  it.hk = rest % a.Hk;
  if (a.inline_list) {
    it.b = rest / a.Hk;
    it.t = 0;
  } else {
    const int2 pr = pairs[rest / a.Hk];
    it.b = pr.x;
    it.t = pr.y;
  }
  it.s = seq_info_l<KL>(a.cu_q, a.keys, it.b);
  it.bad = a.inline_list && !seq_ok<KL>(a, it.b, it.s);
  if (a.inline_list && (it.bad || it.s.lq == 0)) {  // no rows: nothing to load, nothing to write
    it.s.lq = 0;
    it.j0 = it.j1 = 0;
    return it;
  }
  const int nk = fwd_k_tiles((it.t + 1) * a.tq, it.s.lq, it.s.lk, a.causal != 0);
  const int per = (nk + a.splits - 1) / a.splits;
  it.j0 = min(nk, it.split * per);
  it.j1 = min(nk, it.j0 + per);
  return it;
}

// Row of key tile j of the item in the key/value tensor. With an inline list
// the block-table entries have not been checked: a page outside the pool
// gives row 0 and clears `ok`.
template <int KL>
__device__ __forceinline__ int tile_row(const DecodeArgs& a, const Item& it, int j, bool& ok) {
  if (KL != kKeysPaged) return it.s.k0 + j * BN;
  if (!a.inline_list) return key_tile_row(a.keys, it.b, it.s, j);
  const int pos = j * BN;
  const int page = __ldg(a.keys.block_table + static_cast<size_t>(it.b) * a.keys.max_pages + pos / a.keys.page_size);
  if (page < 0 || page >= a.total_k / a.keys.page_size) {
    ok = false;
    return 0;
  }
  return page * a.keys.page_size + pos % a.keys.page_size;
}

template <int D, bool CAUSAL, int KL>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_q3, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const DecodeArgs a) {
  using L = DecSmem<D>;
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
      mbar_init(&bars.o_full[i], 1);
    }
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
    tma_prefetch_desc(&tm_q3);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
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
  const int n_pairs = a.inline_list ? a.batch : static_cast<int>(hdr->n_pairs);
  const int n_items = (hdr->status == FA_OK) ? n_pairs * a.Hk * a.splits : 0;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ Q and K producer
    if (a.inline_list && blockIdx.x == 0) {
      // The whole-batch checks of the work-list kernel: the offsets start at
      // 0 and end at the totals.
      bool ok = __ldg(a.cu_q) == 0 && __ldg(a.cu_q + a.batch) == a.total_q;
      if (KL == kKeysPacked) ok = ok && __ldg(a.keys.cu_k) == 0 && __ldg(a.keys.cu_k + a.batch) == a.total_k;
      if (!ok) atomicCAS(&hdr->status, static_cast<uint32_t>(FA_OK), static_cast<uint32_t>(FA_ERR_BAD_SEQLENS));
    }
    uint32_t kc = 0, nq = 0, ni = 0;
    for (;;) {
      int idx;
      if (!publish_item(bars.items, ni, &hdr->work_counter, n_items, idx, ab)) goto kproducer_done;
      if (idx < 0) break;
      const Item it = get_item<KL>(a, pairs, idx);
      if (it.bad) atomicCAS(&hdr->status, static_cast<uint32_t>(FA_OK), static_cast<uint32_t>(FA_ERR_BAD_SEQLENS));
      if (it.j0 >= it.j1) continue;
      if (nq > 0 && !wait_bar(&bars.q_empty, (nq - 1) & 1, ab)) goto kproducer_done;
      // Rows (token, head): tq tokens from the tile's first, the group's g
      // heads of each (tokens past the tensor end read as zero). When g
      // does not divide 128 the last 128 - g*tq rows are not loaded; they
      // belong to no token and are masked like rows past the sequence.
      mbar_arrive_expect_tx(&bars.q_full, L::kChunks * a.group * a.tq * 128);
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_3d(&tm_q3, &bars.q_full, smem + L::kQ + c * kChunkBytes, c * 64, it.hk * a.group,
                    it.s.q0 + it.t * a.tq);
      ++nq;
      for (int j = it.j0; j < it.j1; ++j, ++kc) {
        const int st = kc % NK;
        const uint32_t use = kc / NK;
        bool page_ok = true;
        const int krow = tile_row<KL>(a, it, j, page_ok);
        if (!page_ok)
          atomicCAS(&hdr->status, static_cast<uint32_t>(FA_OK), static_cast<uint32_t>(FA_ERR_BAD_SEQLENS));
        if (use > 0 && !wait_bar(&bars.k_empty[st], (use - 1) & 1, ab)) goto kproducer_done;
        mbar_arrive_expect_tx(&bars.k_full[st], L::kTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_2d(&tm_k, &bars.k_full[st], smem + L::kK + st * L::kTileBytes + c * kChunkBytes,
                      it.hk * D + c * 64, krow);
      }
    }
  kproducer_done:
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
      const Item it = get_item<KL>(a, pairs, idx);
      for (int j = it.j0; j < it.j1; ++j, ++vc) {
        const int st = vc % NV;
        const uint32_t use = vc / NV;
        bool page_ok = true;  // reported by the K producer
        const int vrow = tile_row<KL>(a, it, j, page_ok);
        if (use > 0 && !wait_bar(&bars.v_empty[st], (use - 1) & 1, ab)) goto vproducer_done;
        mbar_arrive_expect_tx(&bars.v_full[st], L::kTileBytes);
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_2d(&tm_v, &bars.v_full[st], smem + L::kV + st * L::kTileBytes + c * kChunkBytes,
                      it.hk * D + c * 64, vrow);
      }
    }
  vproducer_done:
    for (uint32_t i = (vc > NV ? vc - NV : 0); i < vc; ++i) wait_bar_final(&bars.v_full[i % NV], (i / NV) & 1, ab);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Converged warp, one elected lane issues. Per key tile: S_j = Q K_j^T
    // into S buffer (g + j) & 1, then O (+)= P_{j-1} V_{j-1}; S_{j+1}
    // overwrites P_{j-1} only after that PV was issued (MMAs run in order).
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
      const Item it = get_item<KL>(a, pairs, idx);
      const int nk = it.j1 - it.j0;
      if (nk <= 0) continue;
      if (!wait_bar_warp(&bars.q_full, nq & 1, ab)) goto mma_done;
      tc_fence_after();
      for (int j = 0; j <= nk; ++j) {
        if (j < nk) {
          const uint32_t kvj = kv + j;
          const int st = kvj % NK;
          if (!wait_bar_warp(&bars.k_full[st], (kvj / NK) & 1, ab)) goto mma_done;
          tc_fence_after();
          const uint64_t k_desc = opaque_u64(k_desc0) + static_cast<uint64_t>((st * L::kTileBytes) >> 4);
          const uint32_t d_s = tmem + kSCol + ((g + j) & 1) * BN;
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
              mma_ss(d_s, q_desc + off, k_desc + off, kIdescS, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bars.s_full[(g + j) & 1]);
            mma_commit(&bars.k_empty[st]);
            if (j == nk - 1) mma_commit(&bars.q_empty);
          }
          __syncwarp();
        }
        if (j > 0) {
          const int jj = j - 1;
          const uint32_t gj = g + jj, kvj = kv + jj;
          const int st = kvj % NV;
          if (jj == 0 && nq > 0 && !wait_bar_warp(&bars.o_empty, (nq - 1) & 1, ab)) goto mma_done;
          if (!wait_bar_warp(&bars.v_full[st], (kvj / NV) & 1, ab)) goto mma_done;
          const uint64_t v_desc = opaque_u64(v_desc0) + static_cast<uint64_t>((st * L::kTileBytes) >> 4);
          const uint32_t a_p = tmem + kSCol + (gj & 1) * BN;
          if (!wait_bar_warp(&bars.p_full[gj & 1], (gj >> 1) & 1, ab)) goto mma_done;
          tc_fence_after();
          if (elect_one()) {
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
      kv += nk;
      g += nk;
      ++nq;
    }
  mma_done:
    if (elect_one()) mma_commit(&bars.drain);
    __syncwarp();
    wait_bar_final(&bars.drain, 0, ab);
  } else if (warp >= kSoftmaxWarp0) {
    // ------------------------------------------------------------ softmax and epilogue
    const int m = threadIdx.x - kSoftmaxWarp0 * 32;  // tile row == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_o = tmem + lane_base + kOCol;
    const int mt = m / a.group, mh = m - mt * a.group;  // row m: token mt of the tile, head mh of the group
    uint32_t g = 0, nq = 0, ni = 0;
    for (;;) {
      int slot;
      const int idx = consume_item<true>(bars.items, ni, slot, ab);
      if (idx < 0) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.items.empty[slot]);
      const Item it = get_item<KL>(a, pairs, idx);
      const int h = it.hk * a.group + mh;
      const int r = it.t * a.tq + mt;  // query token within the sequence
      const bool row_ok = mt < a.tq && r < it.s.lq;
      const size_t orow = (static_cast<size_t>(it.s.q0) + r) * a.H + h;  // row of [total_q * H]
      const bool split_out = a.splits > 1;
      const int nk = it.j1 - it.j0;
      float m_used = -INFINITY, l = 0.f;
      const int diag = it.s.lk - it.s.lq;  // key j visible from token i iff j <= i + diag
      for (int jt = 0; jt < nk; ++jt, ++g) {
        const int j = it.j0 + jt;
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
        // Rows past the tile's tokens or the sequence see no key.
        int lim = row_ok ? it.s.lk - key0 : 0;
        if (CAUSAL) lim = min(lim, r + diag + 1 - key0);
        if (__any_sync(0xffffffffu, lim < BN)) {
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
        if (__any_sync(0xffffffffu, jt > 0 && alpha != 1.f)) {
          // The previous PV (global index g-1) must have completed; PV
          // completions alternate between two barriers, so the phase is
          // unambiguous.
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
      {
        // Epilogue. A split with no key tiles (or a row that saw no key)
        // contributes nothing: partial logsumexp -inf and output 0.
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        const float lse_nat = (l > 0.f) ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
        if (nk > 0) {
          if (!wait_bar_warp(&bars.o_full[(g - 1) & 1], ((g - 1) >> 1) & 1, ab)) goto softmax_done;
          tc_fence_after();
        }
        float* op = split_out ? a.opart + (static_cast<size_t>(it.split) * a.total_q * a.H + orow) * D : nullptr;
        uint4* og = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow * D);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (nk > 0) {
            tmem_ld32(t_o + c * 32, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
          }
          if (row_ok) {
            if (split_out) {
#pragma unroll
              for (int e = 0; e < 8; ++e)
                reinterpret_cast<float4*>(op)[c * 8 + e] =
                    make_float4(__uint_as_float(o[4 * e + 0]) * inv, __uint_as_float(o[4 * e + 1]) * inv,
                                __uint_as_float(o[4 * e + 2]) * inv, __uint_as_float(o[4 * e + 3]) * inv);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
                og[c * 4 + e] = w;
              }
            }
          }
        }
        if (row_ok) {
          if (split_out)
            a.lpart[static_cast<size_t>(it.split) * a.total_q * a.H + orow] = lse_nat;
          else
            a.lse[static_cast<size_t>(h) * a.total_q + it.s.q0 + r] = lse_nat;
        }
      }
      if (nk > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.o_empty);
        ++nq;
      }
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

// out = sum_s exp(lse_s - lse) * out_s with lse = log sum_s exp(lse_s), one
// warp per (query token, head) row. The splits are handled 32 at a time:
// lane s loads split s's logsumexp, the maximum and the sum of the weights
// are warp reductions, and the partial outputs (a 16-byte vector per lane at
// d = 128) are loaded eight at a time before any of them is used, so that
// the latency of the partials is paid once per eight splits instead of once
// per split. A split that saw no key (logsumexp -inf, partial written as
// zeros) has weight 0 and is skipped.
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeArgs a) {
  griddep_wait();  // the partials come from the decode kernel before this one
  const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(a.total_q) * a.H;
  if (w >= rows) return;
  const size_t stride = static_cast<size_t>(rows);
  constexpr int E = D / 32;  // channels per lane
  using Vec = typename std::conditional<E == 4, float4, float2>::type;
  static_assert(E == 2 || E == 4, "d = 64 or 128");
  float mx = -INFINITY;
  for (int s0 = 0; s0 < a.splits; s0 += 32)
    if (s0 + lane < a.splits) mx = fmaxf(mx, a.lpart[(s0 + lane) * stride + w]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float sum = 0.f;
  if (mx != -INFINITY) {
    for (int s0 = 0; s0 < a.splits; s0 += 32) {
      const float ls = s0 + lane < a.splits ? a.lpart[(s0 + lane) * stride + w] : -INFINITY;
      const float f = ls == -INFINITY ? 0.f : __expf(ls - mx);
      sum += f;
      const int n = a.splits - s0 < 32 ? a.splits - s0 : 32;
      const float* src = a.opart + ((static_cast<size_t>(s0) * stride + w) * D + lane * E);
      for (int i0 = 0; i0 < n; i0 += 8) {
        // Eight partials in flight before any is used.
        Vec x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (i0 + u < n) x[u] = *reinterpret_cast<const Vec*>(src + static_cast<size_t>(i0 + u) * stride * D);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (i0 + u >= n) break;
          const float fi = __shfl_sync(0xffffffffu, f, i0 + u);
          const float* xv = reinterpret_cast<const float*>(&x[u]);
          if (fi != 0.f) {
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = fmaf(fi, xv[e], acc[e]);
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.out) + w * D + lane * E;
#pragma unroll
  for (int e = 0; e < E; e += 2) *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
  if (lane == 0) {
    const long long row = w / a.H;
    const int h = static_cast<int>(w - row * a.H);
    a.lse[static_cast<size_t>(h) * a.total_q + row] = sum > 0.f ? mx + logf(sum) : -INFINITY;
  }
}

template <int D, bool CAUSAL, int KL>
cudaError_t launch_one(const DecodeArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       cudaStream_t stream) {
  using L = DecSmem<D>;
  auto kern = decode_kernel<D, CAUSAL, KL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, a.grid, kThreads, L::kAlloc, stream, a.chained != 0, tq, tk, tv, a);
}

template <int KL>
cudaError_t launch_layout(const DecodeArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          cudaStream_t stream) {
  if (a.D == 64)
    return a.causal ? launch_one<64, true, KL>(a, tq, tk, tv, stream) : launch_one<64, false, KL>(a, tq, tk, tv, stream);
  return a.causal ? launch_one<128, true, KL>(a, tq, tk, tv, stream) : launch_one<128, false, KL>(a, tq, tk, tv, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          cudaStream_t stream) {
  switch (key_layout(a.keys)) {
    case kKeysPaged: return launch_layout<kKeysPaged>(a, tq, tk, tv, stream);
    case kKeysSlots: return launch_layout<kKeysSlots>(a, tq, tk, tv, stream);
    default: return launch_layout<kKeysPacked>(a, tq, tk, tv, stream);
  }
}

cudaError_t launch_decode_combine(const DecodeArgs& a, cudaStream_t stream) {
  const long long warps = static_cast<long long>(a.total_q) * a.H;
  const unsigned blocks = static_cast<unsigned>((warps + 7) / 8);
  if (blocks == 0 || a.splits <= 1) return cudaSuccess;
  return launch_kernel(a.D == 64 ? decode_combine_kernel<64> : decode_combine_kernel<128>, blocks, 256, 0, stream,
                       a.chained != 0, a);
}

}  // namespace fa
