// fa_kernels.h -- host-side launchers of the library's kernels (private to
// libfa_varlen.so; the public interface is include/fa_varlen.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "fa_common.cuh"

namespace fa {

// Work-list preparation (one CTA): validates the cumulative offsets, counts
// the (sequence, tile) pairs and writes them longest-first into the
// workspace. mode 0: forward query tiles; mode 1: backward key tiles.
struct SchedArgs {
  const int32_t* cu_q;
  KeyRows keys;
  int batch, total_q, total_k, max_seqlen_q, max_seqlen_k;
  int causal;
  int mode;
  int item_rows;      // forward: query rows per work item (fwd_item_rows)
  int natural_order;  // 1: tiles of each sequence in increasing order (tile-major), not longest first
  void* workspace;
  size_t seq_off_offset, pairs_offset;
  int max_pairs;
};
cudaError_t launch_sched_prep(const SchedArgs& a, cudaStream_t stream);

struct FwdArgs {
  const int32_t* cu_q;
  KeyRows keys;
  void* out;         // bf16 [total_q, H, D]
  float* lse;        // fp32 [H, total_q]
  void* workspace;   // header + pairs
  size_t pairs_offset;
  int H, D, total_q;
  int group;         // query heads per key/value head (H / Hk)
  int causal;
  float scale_log2;  // softmax_scale * log2(e)
  int grid;          // persistent CTAs
  uint64_t wait_ns;  // time limit of every pipeline wait
  int withhold_v0;   // test hook: the first V tile load of work item 0 is never issued
  int chained;       // launched as a programmatic dependent of the work-list kernel
};
// tm_q: 2-D map over [rows, H*D] bf16; tm_k / tm_v over [rows, Hk*D]; box
// 128 rows x 64 columns, 128-byte swizzle.
cudaError_t launch_fwd(const FwdArgs& a, const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                       cudaStream_t stream);
// head_dim 256: 128-row query items, 64-key tiles; tm_k / tm_v with boxes of
// 64 rows x 64 columns.
cudaError_t launch_fwd_d256(const FwdArgs& a, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                            const CUtensorMap& tm_v, cudaStream_t stream);

// Split-KV forward with the query heads of a key/value group packed into
// the rows of one tile (the decode path): an item is (sequence, key/value
// head, tile of tq = 128 / group query tokens, key split); its 128 rows are
// (token, head-in-group) pairs. With splits > 1 every split writes a
// normalised partial output and its logsumexp (fp32) and the combine kernel
// merges them. tm_q3: 3-D map over q as [tokens, H, D] with box (64, group,
// tq); tm_k / tm_v as for launch_fwd.
struct DecodeArgs {
  const int32_t* cu_q;
  KeyRows keys;
  void* out;        // bf16 [total_q, H, D]
  float* lse;       // fp32 [H, total_q]
  float* opart;     // fp32 [splits, total_q * H, D] (splits > 1)
  float* lpart;     // fp32 [splits, total_q * H]    (splits > 1)
  void* workspace;  // header + pairs
  size_t pairs_offset;
  int H, Hk, group, D, total_q;
  int tq;           // query tokens per item
  int splits;
  int causal;
  float scale_log2;
  int grid;
  uint64_t wait_ns;  // time limit of every pipeline wait
  int chained;       // decode chained to the work-list kernel, combine to decode
  // 1: no work list. Every sequence has at most one query tile, so item idx
  // is (sequence idx / (Hk * splits), its only tile); the kernel checks each
  // item's sequence itself (the checks of the work-list kernel) and the
  // call resets the header instead of running that kernel.
  int inline_list;
  int batch, total_k, max_seqlen_q, max_seqlen_k;
};
cudaError_t launch_decode(const DecodeArgs& a, const CUtensorMap& tm_q3, const CUtensorMap& tm_k,
                          const CUtensorMap& tm_v, cudaStream_t stream);
cudaError_t launch_decode_combine(const DecodeArgs& a, cudaStream_t stream);

struct BwdArgs {
  const int32_t* cu_q;
  KeyRows keys;      // packed layout only
  const void* dout;   // bf16 [total_q, H, D]
  const void* out;    // bf16 [total_q, H, D]
  const float* lse;   // fp32 [H, total_q]
  void* dq;           // bf16 [total_q, H, D]
  void* dk;           // bf16 [total_k, H, D]
  void* dv;           // bf16 [total_k, H, D]
  void* workspace;
  size_t pairs_offset, dvec_offset, qcount_offset, dqacc_offset;
  int deterministic;  // add dQ contributions in key-tile order (bitwise reproducible)
  int tq_pad;
  int H, D, total_q, total_k;  // H: query heads
  int Hk, group;               // key/value heads, query heads per key/value head
  int causal;
  float scale;        // softmax_scale
  float scale_log2;   // softmax_scale * log2(e)
  int grid;
  uint64_t wait_ns;   // time limit of every pipeline wait
  int chained;        // each launch a programmatic dependent of the one before it
};
// Backward in three launches: preprocess (rowsum(dO*O) and zero the dQ
// accumulator), main, dQ conversion. Tensor maps, all bf16 with 128-byte
// swizzle and 64-column boxes: q / dout over [rows, H*D] with 128-row boxes
// (loads); k / v over [rows, Hk*D] with 128-row boxes (loads); dk / dv over
// [rows, Hk*D] with 128-row boxes (stores of whole key tiles).
// At head_dim 64 dQ leaves through tensor reductions: dqacc is an fp32 map
// over the accumulator viewed as [H * tq_pad rows, 64], boxes of 128 rows x
// 32 columns (128 bytes) with 128-byte swizzle (unused at head_dim 128).
struct BwdMaps {
  CUtensorMap q, k, v, dout, dk, dv, dqacc;
};
// head_dim 256: a dV pass (q / dout maps with 128-row boxes) and a dK/dQ
// pass (q / dout maps with 64-row boxes); k, v with 128-row boxes. Both take
// the same work list; the second uses the header's second work counter.
struct BwdMapsD256 {
  CUtensorMap q128, do128, q64, do64, k, v;
};
cudaError_t launch_bwd_d256(const BwdArgs& a, const BwdMapsD256& maps, cudaStream_t stream);
cudaError_t launch_bwd_preprocess(const BwdArgs& a, cudaStream_t stream);
cudaError_t launch_bwd_main(const BwdArgs& a, const BwdMaps& maps, cudaStream_t stream);
cudaError_t launch_bwd_convert(const BwdArgs& a, cudaStream_t stream);

}  // namespace fa
