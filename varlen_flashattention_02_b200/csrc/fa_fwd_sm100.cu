// fa_fwd_sm100.cu -- forward varlen attention for sm_100a.
//
// One persistent CTA per SM takes (sequence, head, 256-row query block)
// items from the scheduler's longest-first list through a global counter.
// An item is computed as two query tiles of 128 rows that share every key
// and value tile. For each tile, exact attention over the sequence's keys
// with an online softmax:
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
//  * warp specialisation (16 warps): warp 0 issues the Q and K TMA loads and
//    hands out work items, warp 2 the V loads (separate rings, so K can run
//    ahead of V), warp 1 issues the tcgen05 MMAs; warpgroups 1 and 2 (one
//    thread per query row and TMEM lane) run the softmax of query tile 0 and
//    of query tile 1; warpgroup 3 normalises O and stores it. This is the
//    pages' split of Q across workers that share K and V, at warpgroup
//    granularity: while one softmax warpgroup works, the tensor pipe runs the
//    other tile's P V and next Q K^T, so the softmax latency hides behind
//    MMAs, and each K/V tile loaded serves 256 query rows;
//  * accumulators live in tensor memory: S_0, S_1 (one per query tile), O_0,
//    O_1. P overwrites its own S columns as bf16 and feeds the PV MMA
//    directly from TMEM; MMAs run in issue order, so the next Q K^T of a
//    tile, issued after its PV, may overwrite P;
//  * O is rescaled only when a row maximum grows by more than 2^8 (the
//    stale maximum stays consistent with l, so the result is exact);
//  * masking is applied only on the last key tile of a sequence and on
//    tiles that cross the causal diagonal; tiles wholly above it are never
//    loaded;
//  * grouped- and multi-query attention ("Flash-Atención y Flash-Atención-2",
//    FlashAttention-2 section): query head h reads key/value head
//    h / (H / Hk); items of consecutive query heads are adjacent in the work
//    order, so a shared K/V tile is usually still in L2 for the next one.
#include "fa_common.cuh"
#include "fa_kernels.h"

namespace fa {
namespace {

constexpr int BM = kFwdBM;
constexpr int BN = kFwdBN;
constexpr int kQTiles = kFwdItemRows / kFwdBM;
static_assert(kQTiles == 2, "one softmax warpgroup per query tile, two of them");
constexpr int kThreads = 512;
constexpr int kSoftmaxWarp0 = 4;    // warps 4-7: query tile 0, warps 8-11: query tile 1
constexpr int kEpilogueWarp0 = 12;  // warps 12-15
constexpr int kChunkBytes = 128 * 128;  // one [128 rows x 64 bf16] swizzled chunk
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Registers per thread. 512 threads start with 128 each (the whole 64K
// register file); the load/MMA and epilogue warpgroups give registers to
// the softmax warpgroups, which hold a 128-column row of S. The shares add
// up to exactly the file, so both increases are always satisfied.
constexpr uint32_t kRegsLaunch = 128, kRegsLoad = 80, kRegsSoftmax = 184, kRegsEpilogue = 64;
static_assert(kRegsLoad + 2 * kRegsSoftmax + kRegsEpilogue == 4 * kRegsLaunch, "register split uses the launch's file");

template <int D>
struct FwdSmem {
  // K and V have rings of their own: a K stage is released as soon as the
  // Q K^T of both query tiles have read it, a V stage only after both PVs.
  static constexpr int kKStages = (D == 64) ? 5 : 3;
  static constexpr int kVStages = (D == 64) ? 5 : 2;
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;  // Q, K or V tile
  static constexpr int kQ = 0;                              // query tile w at kQ + w*tile
  static constexpr int kK = kQ + kQTiles * kTileBytes;      // K stage s at kK + s*tile
  static constexpr int kV = kK + kKStages * kTileBytes;     // V stage s at kV + s*tile
  static constexpr int kInvL = kV + kVStages * kTileBytes;  // fp32 [2][128]: 1/l per row
  static constexpr int kBar = kInvL + kQTiles * BM * 4;
  static constexpr int kBytes = kBar + 1024;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  static constexpr int kSCol = 0;               // S of query tile w at columns w*BN
  static constexpr int kOCol = 2 * BN;          // O of query tile w at kOCol + w*D
};
static_assert(FwdSmem<128>::kAlloc <= 232448 && FwdSmem<64>::kAlloc <= 232448, "layout fits 227 KB");

struct Item {
  int b, h, t;  // t: 256-row block of the sequence
  int hk;       // key/value head of query head h
  SeqInfo s;
  int nk[2];    // key tiles visible from query tile w (0 when the tile is empty)
};

// Decoded items travel through the item ring at head_dim 128 (the
// producer decodes each item once and the other roles copy it); at head_dim
// 64 every role decodes the index itself, which measured faster there.
template <int D>
constexpr bool kDecodedRing = D != 64;

struct Bars {
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], p_full[2];
  uint64_t o_full[2], o_empty[2];
  uint64_t l_full[2], l_empty[2];
  uint64_t drain;
  uint64_t k_full[5], k_empty[5], v_full[5], v_empty[5];
  ItemRing items;
  Item item_data[kItemSlots];  // the published items, decoded once by the producer
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 1024, "barrier block fits its reserved space");

template <int KL>
__device__ __forceinline__ Item get_item(const FwdArgs& a, const int2* pairs, int idx) {
  Item it;
  const int2 pr = pairs[idx / a.H];
  it.h = idx % a.H;
  it.hk = it.h / a.group;
  it.b = pr.x;
  it.t = pr.y;
  it.s = seq_info_l<KL>(a.cu_q, a.keys, it.b);
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const int row0 = (it.t * kQTiles + w) * BM;
    it.nk[w] = row0 < it.s.lq ? fwd_k_tiles(row0 + BM, it.s.lq, it.s.lk, a.causal != 0) : 0;
  }
  return it;
}

// ---------------------------------------------------------------- roles
// Each role is inlined into the kernel: code after a register reallocation
// may not call out-of-line functions.

// KL: the key layout (packed, cache slots, pages), a compile-time choice:
// code for the other layouts in these loops slows them measurably.
template <int D, int KL>
__device__ __forceinline__ void qk_producer(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const FwdArgs& a,
                                            uint8_t* smem, Bars& bars, WsHeader* hdr, const int2* pairs,
                                            int n_items, const Abort& ab) {
  using L = FwdSmem<D>;
  constexpr int NK = L::kKStages;
  uint32_t kc = 0, ni = 0, nq[2] = {0u, 0u};
  for (;;) {
    int idx;
    Item it;
    if constexpr (kDecodedRing<D>) {
      auto decode = [&](int slot, int v) {
        it = get_item<KL>(a, pairs, v);
        bars.item_data[slot] = it;
      };
      if (!publish_item_decoded(bars.items, ni, &hdr->work_counter, n_items, idx, ab, decode)) goto done;
    } else {
      if (!publish_item(bars.items, ni, &hdr->work_counter, n_items, idx, ab)) goto done;
      if (idx >= 0) it = get_item<KL>(a, pairs, idx);
    }
    if (idx < 0) break;
    const int nkb = max(it.nk[0], it.nk[1]);
    if (nkb == 0) continue;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      if (it.nk[w] == 0) continue;
      if (nq[w] > 0 && !wait_bar(&bars.q_empty[w], (nq[w] - 1) & 1, ab)) goto done;
      mbar_arrive_expect_tx(&bars.q_full[w], L::kTileBytes);
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_2d(tm_q, &bars.q_full[w], smem + L::kQ + w * L::kTileBytes + c * kChunkBytes, it.h * D + c * 64,
                    it.s.q0 + (it.t * kQTiles + w) * BM);
      ++nq[w];
    }
    for (int j = 0; j < nkb; ++j, ++kc) {
      const int st = kc % NK;
      const uint32_t use = kc / NK;
      // A block-table read for a paged cache, issued before the stage wait.
      const int krow = KL == kKeysPaged ? key_tile_row(a.keys, it.b, it.s, j) : it.s.k0 + j * BN;
      if (use > 0 && !wait_bar(&bars.k_empty[st], (use - 1) & 1, ab)) goto done;
      mbar_arrive_expect_tx(&bars.k_full[st], L::kTileBytes);
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_2d(tm_k, &bars.k_full[st], smem + L::kK + st * L::kTileBytes + c * kChunkBytes,
                    it.hk * D + c * 64, krow);
    }
  }
done:
  // Never leave TMA writes in flight into shared memory that is about to be
  // given up: wait (bounded) for the last loads issued.
  for (int w = 0; w < 2; ++w)
    if (nq[w] > 0) wait_bar_final(&bars.q_full[w], (nq[w] - 1) & 1, ab);
  for (uint32_t i = (kc > NK ? kc - NK : 0); i < kc; ++i) wait_bar_final(&bars.k_full[i % NK], (i / NK) & 1, ab);
}

template <int D, int KL>
__device__ __forceinline__ void v_producer(const CUtensorMap* tm_v, const FwdArgs& a, uint8_t* smem, Bars& bars,
                                           const int2* pairs, const Abort& ab) {
  using L = FwdSmem<D>;
  constexpr int NV = L::kVStages;
  uint32_t vc = 0, ni = 0;
  uint32_t withheld = 0xffffffffu;  // test hook: the V load that was never issued
  for (;;) {
    int slot;
    const int idx = consume_item<false>(bars.items, ni, slot, ab);
    if (idx < 0) break;
    const Item it = kDecodedRing<D> ? bars.item_data[slot] : get_item<KL>(a, pairs, idx);
    mbar_arrive(&bars.items.empty[slot]);
    const int nkb = max(it.nk[0], it.nk[1]);
    for (int j = 0; j < nkb; ++j, ++vc) {
      const int st = vc % NV;
      const uint32_t use = vc / NV;
      const int vrow = KL == kKeysPaged ? key_tile_row(a.keys, it.b, it.s, j) : it.s.k0 + j * BN;
      if (use > 0 && !wait_bar(&bars.v_empty[st], (use - 1) & 1, ab)) goto done;
      if (a.withhold_v0 && idx == 0 && j == 0) {
        // Test hook: neither the load nor its expected bytes are posted, so
        // the MMA warp's wait for this stage runs out (nothing is left in
        // flight) and the CTA reports FA_ERR_DEVICE_TIMEOUT.
        withheld = vc;
        continue;
      }
      mbar_arrive_expect_tx(&bars.v_full[st], L::kTileBytes);
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_2d(tm_v, &bars.v_full[st], smem + L::kV + st * L::kTileBytes + c * kChunkBytes,
                    it.hk * D + c * 64, vrow);
    }
  }
done:
  for (uint32_t i = (vc > NV ? vc - NV : 0); i < vc; ++i)
    if (i != withheld) wait_bar_final(&bars.v_full[i % NV], (i / NV) & 1, ab);
}

// The MMA issuer. The whole warp runs this loop converged (all values
// warp-uniform); one elected lane issues each group of MMAs and the commits.
// Shared memory descriptors are built once and advanced by constant offsets.
//
// Order per key tile j, for query tile w = 0 then 1 (when the tile sees key
// tile j): wait for P_w,j; O_w (+)= P_w,j V_j; S_w,j+1 = Q_w K_{j+1}^T.
// The two tiles' softmax phases are thereby offset: while warpgroup w works
// on S_w,j+1, the tensor pipe runs the other tile's PV and Q K^T.
template <int D, int KL>
__device__ __forceinline__ void mma_issuer(const FwdArgs& a, uint8_t* smem, Bars& bars, const int2* pairs,
                                           uint32_t tmem, const Abort& ab) {
  using L = FwdSmem<D>;
  constexpr int NK = L::kKStages, NV = L::kVStages;
  constexpr uint32_t kIdescS = idesc_bf16_f32(BM, BN, false, false);
  constexpr uint32_t kIdescO = idesc_bf16_f32(BM, D, false, true);
  const uint64_t q_desc0 = smem_desc_sw128(smem_u32(smem + L::kQ), 16, 1024);
  const uint64_t k_desc0 = smem_desc_sw128(smem_u32(smem + L::kK), 16, 1024);
  const uint64_t v_desc0 = smem_desc_sw128(smem_u32(smem + L::kV), kChunkBytes, 1024);
  uint32_t kv = 0, ni = 0;
  uint32_t nq[2] = {0u, 0u};  // items so far in which query tile w had work
  uint32_t np[2] = {0u, 0u};  // P tiles consumed so far, per query tile

  // S_w = Q_w K^T from K stage st.
  auto issue_s = [&](int w, int st) {
    const uint64_t q_desc = opaque_u64(q_desc0) + static_cast<uint64_t>((w * L::kTileBytes) >> 4);
    const uint64_t k_desc = opaque_u64(k_desc0) + static_cast<uint64_t>((st * L::kTileBytes) >> 4);
    const uint32_t d_s = tmem + L::kSCol + w * BN;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
      mma_ss(d_s, q_desc + off, k_desc + off, kIdescS, kk > 0 ? 1u : 0u);
    }
  };

  for (;;) {
    int slot;
    const int idx = consume_item<true>(bars.items, ni, slot, ab);
    if (idx < 0) break;
    const Item it = kDecodedRing<D> ? bars.item_data[slot] : get_item<KL>(a, pairs, idx);
    __syncwarp();
    if (elect_one()) mbar_arrive(&bars.items.empty[slot]);
    __syncwarp();
    const int nkb = max(it.nk[0], it.nk[1]);
    if (nkb == 0) continue;
#pragma unroll
    for (int w = 0; w < 2; ++w)
      if (it.nk[w] > 0 && !wait_bar_warp(&bars.q_full[w], nq[w] & 1, ab)) goto done;
    {
      // S_w,0 for both query tiles.
      const int st = kv % NK;
      if (!wait_bar_warp(&bars.k_full[st], (kv / NK) & 1, ab)) goto done;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (it.nk[w] == 0) continue;
          issue_s(w, st);
          mma_commit(&bars.s_full[w]);
          if (it.nk[w] == 1) mma_commit(&bars.q_empty[w]);
        }
        mma_commit(&bars.k_empty[st]);
      }
      __syncwarp();
    }
    for (int j = 0; j < nkb; ++j) {
      const uint32_t kvj = kv + j;
      const int vst = kvj % NV;
      const int kst = (kvj + 1) % NK;  // stage of key tile j+1
      bool k_ready = false;
      if (!wait_bar_warp(&bars.v_full[vst], (kvj / NV) & 1, ab)) goto done;
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        if (j >= it.nk[w]) continue;
        if (j == 0 && nq[w] > 0 && !wait_bar_warp(&bars.o_empty[w], (nq[w] - 1) & 1, ab)) goto done;
        const bool more = j + 1 < it.nk[w];
        if (more && !k_ready) {
          if (!wait_bar_warp(&bars.k_full[kst], ((kvj + 1) / NK) & 1, ab)) goto done;
          k_ready = true;
        }
        // O_w (+)= P_w V_j with P read from TMEM, then S_w,j+1. Everything
        // that does not depend on P (the waits above, the descriptors) is
        // done before waiting for it, so the MMAs issue as soon as P lands.
        const uint64_t v_desc = opaque_u64(v_desc0) + static_cast<uint64_t>((vst * L::kTileBytes) >> 4);
        const uint32_t a_p = tmem + L::kSCol + w * BN;
        const uint32_t d_o = tmem + L::kOCol + w * D;
        if (!wait_bar_warp(&bars.p_full[w], np[w] & 1, ab)) goto done;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk)
            mma_ts(d_o, a_p + kk * 8, v_desc + static_cast<uint64_t>((kk * 2048) >> 4), kIdescO,
                   (j > 0 || kk > 0) ? 1u : 0u);
          if (more) {
            issue_s(w, kst);
            mma_commit(&bars.s_full[w]);
            if (j + 2 == it.nk[w]) mma_commit(&bars.q_empty[w]);
          } else {
            mma_commit(&bars.o_full[w]);
          }
        }
        __syncwarp();
        ++np[w];
      }
      if (elect_one()) {
        mma_commit(&bars.v_empty[vst]);
        if (k_ready) mma_commit(&bars.k_empty[kst]);
      }
      __syncwarp();
    }
    kv += nkb;
#pragma unroll
    for (int w = 0; w < 2; ++w) nq[w] += it.nk[w] > 0 ? 1u : 0u;
  }
done:
  // Make sure every MMA this warp issued has finished before TMEM is freed.
  if (elect_one()) mma_commit(&bars.drain);
  __syncwarp();
  wait_bar_final(&bars.drain, 0, ab);
}

// Softmax of query tile W (warps 4+4W .. 7+4W, one thread per row).
template <int D, bool CAUSAL, int W, int KL>
__device__ __forceinline__ void softmax_role(const FwdArgs& a, uint8_t* smem, Bars& bars, const int2* pairs,
                                             uint32_t tmem, const Abort& ab, int warp, int lane) {
  using L = FwdSmem<D>;
  const int row = static_cast<int>(threadIdx.x) - (kSoftmaxWarp0 + 4 * W) * 32;  // row in tile == TMEM lane
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const uint32_t t_s = tmem + lane_base + L::kSCol + W * BN;
  const uint32_t t_o = tmem + lane_base + L::kOCol + W * D;
  float* inv_l_smem = reinterpret_cast<float*>(smem + L::kInvL) + W * BM;
  uint32_t g = 0, nl = 0, ni = 0;
  for (;;) {
    int slot;
    const int idx = consume_item<true>(bars.items, ni, slot, ab);
    if (idx < 0) break;
    const Item it = kDecodedRing<D> ? bars.item_data[slot] : get_item<KL>(a, pairs, idx);
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.items.empty[slot]);
    const int nk = it.nk[W];
    if (nk == 0) continue;  // the epilogue warpgroup writes empty rows
    const int tq = it.t * kQTiles + W;  // 128-row tile of the sequence
    const int r = tq * BM + row;        // row within the sequence
    float m_used = -INFINITY, l = 0.f;
    const int diag = it.s.lk - it.s.lq;  // key j visible from row i iff j <= i + diag
    for (int j = 0; j < nk; ++j, ++g) {
      if (!wait_bar_warp(&bars.s_full[W], g & 1, ab)) return;
      tc_fence_after();
      uint32_t sr[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tmem_ld32(t_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      float* s = reinterpret_cast<float*>(sr);
      const int key0 = j * BN;
      const bool need_mask = (key0 + BN > it.s.lk) || (CAUSAL && key0 + BN - 1 > tq * BM + diag);
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
        // S_j complete implies that the PV of tile j-1 has completed too: the
        // MMA warp issued it before this S, and a commit tracks every earlier
        // MMA of the issuing thread. O stays put until P_j is handed over.
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
      // p = exp2(s * scale * log2e - m): pairs of columns share one packed
      // FMA and one packed add into the partial row sums. P (bf16, two per
      // column) overwrites the first BN/2 columns of S, 32 keys at a time.
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
      // Hand P over first; the row sum is reduced afterwards, off the path
      // to the next MMAs.
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[W]);
      {
        float a0, a1, b0, b1;
        f2_split(f2_add(ls2[0], ls2[1]), a0, a1);
        f2_split(f2_add(ls2[2], ls2[3]), b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
    }
    // Hand 1/l to the epilogue warpgroup; write the LSE of valid rows.
    if (nl > 0 && !wait_bar_warp(&bars.l_empty[W], (nl - 1) & 1, ab)) return;
    inv_l_smem[row] = (l > 0.f) ? 1.f / l : 0.f;
    mbar_arrive(&bars.l_full[W]);
    if (r < it.s.lq)
      a.lse[static_cast<size_t>(it.h) * a.total_q + it.s.q0 + r] =
          (l > 0.f) ? (m_used + log2f(l)) * 0.69314718055994531f : -INFINITY;
    ++nl;
  }
}

// Epilogue (warps 12-15, one thread per row): out = O / l for both query
// tiles of every item, zero rows for tiles that see no key.
template <int D, int KL>
__device__ __forceinline__ void epilogue_role(const FwdArgs& a, uint8_t* smem, Bars& bars, const int2* pairs,
                                              uint32_t tmem, const Abort& ab, int warp, int lane) {
  using L = FwdSmem<D>;
  const int row = static_cast<int>(threadIdx.x) - kEpilogueWarp0 * 32;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  const float* inv_l_smem = reinterpret_cast<const float*>(smem + L::kInvL);
  uint32_t ni = 0, nl[2] = {0u, 0u};
  for (;;) {
    int slot;
    const int idx = consume_item<true>(bars.items, ni, slot, ab);
    if (idx < 0) break;
    const Item it = kDecodedRing<D> ? bars.item_data[slot] : get_item<KL>(a, pairs, idx);
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars.items.empty[slot]);
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int r = (it.t * kQTiles + w) * BM + row;
      const bool row_ok = r < it.s.lq;
      const size_t orow = (static_cast<size_t>(it.s.q0) + r) * a.H + it.h;
      uint4* o_g = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + orow * D);
      if (it.nk[w] == 0) {
        if (row_ok) {
#pragma unroll
          for (int c = 0; c < D / 8; ++c) o_g[c] = make_uint4(0, 0, 0, 0);
          a.lse[static_cast<size_t>(it.h) * a.total_q + it.s.q0 + r] = -INFINITY;
        }
        continue;
      }
      if (!wait_bar_warp(&bars.l_full[w], nl[w] & 1, ab)) return;
      const float inv = inv_l_smem[w * BM + row];
      mbar_arrive(&bars.l_empty[w]);
      if (!wait_bar_warp(&bars.o_full[w], nl[w] & 1, ab)) return;
      tc_fence_after();
      const uint32_t t_o = tmem + lane_base + L::kOCol + w * D;
#pragma unroll 1
      for (int c = 0; c < D / 16; ++c) {
        uint32_t o[16];
        tmem_ld16(t_o + c * 16, o);
        tmem_wait_ld();
        if (c == D / 16 - 1) {
          // O_w has been read: the next item's first PV may overwrite it.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.o_empty[w]);
        }
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
            v.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
            v.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
            v.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
            o_g[c * 2 + e] = v;
          }
        }
      }
      ++nl[w];
    }
  }
}

// End of every warpgroup's branch: once all 512 threads are done with TMEM,
// warp 1 frees it. A named barrier, as the four branches reach it from
// different places.
__device__ __forceinline__ void teardown(uint32_t tmem, int warp) {
  tc_fence_before();
  named_bar_sync(1, kThreads);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool CAUSAL, int KL>
__global__ void __launch_bounds__(kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  using L = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars& bars = *reinterpret_cast<Bars*>(smem + L::kBar);

  auto* hdr = reinterpret_cast<WsHeader*>(a.workspace);
  const int2* pairs = reinterpret_cast<const int2*>(static_cast<const char*>(a.workspace) + a.pairs_offset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars.q_full[w], 1);
      mbar_init(&bars.q_empty[w], 1);
      mbar_init(&bars.s_full[w], 1);
      mbar_init(&bars.p_full[w], 4);
      mbar_init(&bars.o_full[w], 1);
      mbar_init(&bars.o_empty[w], 4);
      mbar_init(&bars.l_full[w], BM);
      mbar_init(&bars.l_empty[w], BM);
    }
    mbar_init(&bars.drain, 1);
    for (int i = 0; i < L::kKStages; ++i) {
      mbar_init(&bars.k_full[i], 1);
      mbar_init(&bars.k_empty[i], 1);
    }
    for (int i = 0; i < L::kVStages; ++i) {
      mbar_init(&bars.v_full[i], 1);
      mbar_init(&bars.v_empty[i], 1);
    }
    // Item consumers: V producer (1), MMA warp (1), softmax warps (8),
    // epilogue warps (4).
    item_ring_init(bars.items, 14);
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

  // Warpgroup index broadcast from lane 0 so that the compiler sees a
  // warp-uniform branch around the register reallocation. Registers move
  // only once, at the start: the load/MMA and epilogue warpgroups release
  // theirs (which never waits), and the softmax warpgroups' increases wait
  // for exactly those. No warpgroup takes registers back at the end: one
  // that finished early could otherwise take registers that a softmax
  // warpgroup has not yet claimed, and that increase would wait forever.
  const int wgroup = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) / 128, 0);
  if (wgroup == 0) {
    warpgroup_reg_dealloc<kRegsLoad>();
    if (warp == 0) {
      if (lane == 0) qk_producer<D, KL>(&tm_q, &tm_k, a, smem, bars, hdr, pairs, n_items, ab);
    } else if (warp == 1) {
      mma_issuer<D, KL>(a, smem, bars, pairs, tmem, ab);
    } else if (warp == 2) {
      if (lane == 0) v_producer<D, KL>(&tm_v, a, smem, bars, pairs, ab);
    }
    __syncwarp();
    teardown(tmem, warp);
  } else if (wgroup == 1) {
    warpgroup_reg_alloc<kRegsSoftmax>();
    softmax_role<D, CAUSAL, 0, KL>(a, smem, bars, pairs, tmem, ab, warp, lane);
    __syncwarp();
    teardown(tmem, warp);
  } else if (wgroup == 2) {
    warpgroup_reg_alloc<kRegsSoftmax>();
    softmax_role<D, CAUSAL, 1, KL>(a, smem, bars, pairs, tmem, ab, warp, lane);
    __syncwarp();
    teardown(tmem, warp);
  } else {
    warpgroup_reg_dealloc<kRegsEpilogue>();
    epilogue_role<D, KL>(a, smem, bars, pairs, tmem, ab, warp, lane);
    __syncwarp();
    teardown(tmem, warp);
  }
}

template <int D, bool CAUSAL, int KL>
cudaError_t launch_one(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       cudaStream_t stream) {
  using L = FwdSmem<D>;
  auto kern = fwd_kernel<D, CAUSAL, KL>;
  // The warpgroups' register shares add up to exactly the launch's 128 per
  // thread; with any other count an increase could wait forever.
  static const int launch_regs = [&] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : -1;
  }();
  if (launch_regs != static_cast<int>(kRegsLaunch)) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, a.grid, kThreads, L::kAlloc, stream, a.chained != 0, tq, tk, tv, a);
}

template <int KL>
cudaError_t launch_layout(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                          cudaStream_t stream) {
  if (a.D == 64)
    return a.causal ? launch_one<64, true, KL>(a, tq, tk, tv, stream)
                    : launch_one<64, false, KL>(a, tq, tk, tv, stream);
  return a.causal ? launch_one<128, true, KL>(a, tq, tk, tv, stream)
                  : launch_one<128, false, KL>(a, tq, tk, tv, stream);
}

}  // namespace

cudaError_t launch_fwd(const FwdArgs& a, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       cudaStream_t stream) {
  switch (key_layout(a.keys)) {
    case kKeysPaged: return launch_layout<kKeysPaged>(a, tq, tk, tv, stream);
    case kKeysSlots: return launch_layout<kKeysSlots>(a, tq, tk, tv, stream);
    default: return launch_layout<kKeysPacked>(a, tq, tk, tv, stream);
  }
}

}  // namespace fa
