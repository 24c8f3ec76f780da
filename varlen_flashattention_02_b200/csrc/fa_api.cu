// fa_api.cu -- the C ABI of libfa_varlen.so (declared in include/fa_varlen.h):
// argument validation, workspace layout, TMA descriptor encoding and kernel
// launches. Host code only; it never synchronises except in
// fa_get_device_status.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fa_varlen.h"
#include "fa_common.cuh"
#include "fa_kernels.h"

namespace {

using fa::WsLayout;

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 map over a packed [rows, H*D] tensor: inner dimension H*D
// elements, row stride H*D*2 bytes, box = 64 columns x box_rows rows,
// 128-byte swizzle, out-of-range rows read as zero.
bool encode_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D bf16 map over q viewed as [tokens, H, D]: box = 64 channels x g heads x
// tq tokens, 128-byte swizzle; it lands the (token, head) rows of a group
// as consecutive 128-byte rows.
// fp32 2-D map [rows, cols] with boxes of 128 rows x 32 columns (128 bytes),
// 128-byte swizzle: the backward's dQ accumulator at head_dim 64.
bool encode_map_f32(CUtensorMap* map, const void* base, long long rows, int cols) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
  cuuint32_t box[2] = {32, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_map_q3(CUtensorMap* map, const void* base, int tokens, int H, int D, int g, int tq) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(g), static_cast<cuuint32_t>(tq)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Measurement hook state (per host thread): events recorded around each
// kernel launch of the next calls.
struct KernelEvents {
  void* const* events = nullptr;
  int n_pairs = 0;
  int next = 0;
};
thread_local KernelEvents t_events;

// Test hooks (per host thread): the wait limit of the kernels and the
// withheld value load of fa_set_test_hooks.
struct TestHooks {
  uint64_t wait_ns = fa::kWaitTimeoutNs;
  int withhold_v0 = 0;
};
thread_local TestHooks t_hooks;

// Runs one launch, bracketed by the caller's timing events when the hook is on.
template <class F>
cudaError_t timed_launch(cudaStream_t stream, F&& launch) {
  KernelEvents& ev = t_events;
  const int i = ev.next++;
  const bool on = ev.events && i < ev.n_pairs;
  if (on && cudaEventRecord(static_cast<cudaEvent_t>(ev.events[2 * i]), stream) != cudaSuccess) return cudaErrorUnknown;
  cudaError_t e = launch();
  if (e != cudaSuccess) return e;
  if (on && cudaEventRecord(static_cast<cudaEvent_t>(ev.events[2 * i + 1]), stream) != cudaSuccess)
    return cudaErrorUnknown;
  return cudaSuccess;
}

// Each kernel of a call after the work-list kernel is launched as a
// programmatic dependent of the one before it (its launch and prologue
// overlap that kernel's tail), except while the per-kernel timing hook is
// on: its events sit between the launches and time each kernel alone.
bool chained() { return t_events.events == nullptr; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Shared size checks of both directions.
fa_status_t check_sizes(int batch, int total_q, int total_k, int max_sq, int max_sk, int H, int Hk, int D,
                        float scale) {
  if (batch < 1 || total_q < 0 || total_k < 0 || max_sq < 0 || max_sk < 0 || H < 1) return FA_ERR_INVALID_ARGUMENT;
  if (Hk < 1 || Hk > H || H % Hk != 0) return FA_ERR_INVALID_ARGUMENT;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARGUMENT;
  if (D != 64 && D != 128 && D != 256) return FA_ERR_UNSUPPORTED;
  // Row indices and TMA coordinates are int32; element offsets are 64-bit.
  const long long hd = static_cast<long long>(H) * D;
  if (hd > (1ll << 31) - 1 || static_cast<long long>(total_q) + 2 * fa::kFwdBM > (1ll << 31) - 1 ||
      static_cast<long long>(total_k) + 2 * fa::kFwdBN > (1ll << 31) - 1)
    return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(total_q / fa::kFwdBM + batch + 1) * H > (1ll << 31) - 1 ||
      static_cast<long long>(total_k / fa::kBwdBN + batch + 1) * H > (1ll << 31) - 1)
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// The forward for either key layout. total_k: rows of the key/value tensors.
fa_status_t run_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q, const fa::KeyRows& keys,
                    int batch, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int num_heads,
                    int num_heads_k, int head_dim, float softmax_scale, int causal, void* out, float* softmax_lse,
                    void* workspace, size_t workspace_bytes, fa_cuda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  fa_status_t st = check_sizes(batch, total_q, total_k, max_seqlen_q, max_seqlen_k, num_heads, num_heads_k,
                               head_dim, softmax_scale);
  if (st != FA_OK) return st;
  if (!cu_seqlens_q) return FA_ERR_INVALID_ARGUMENT;
  if (total_q > 0 && (!q || !out || !softmax_lse || !aligned16(q) || !aligned16(out))) return FA_ERR_INVALID_ARGUMENT;
  if (total_k > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return FA_ERR_INVALID_ARGUMENT;
  const WsLayout L = fa::ws_layout(false, batch, total_q, total_k, num_heads, head_dim);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < L.total)
    return FA_ERR_WORKSPACE;

  t_events.next = 0;
  fa::SchedArgs sa{cu_seqlens_q, keys, batch, total_q, total_k, max_seqlen_q, max_seqlen_k,
                   causal ? 1 : 0, 0, fa::fwd_item_rows(head_dim), 0, workspace, L.seq_off, L.pairs, L.max_pairs};
  if (timed_launch(stream, [&] { return fa::launch_sched_prep(sa, stream); }) != cudaSuccess) return FA_ERR_CUDA;
  if (total_q == 0) return FA_OK;

  const int HD = num_heads * head_dim;
  const int HkD = num_heads_k * head_dim;
  CUtensorMap tq, tk, tv;
  // With no keys at all every row is empty and K/V are never read; the maps
  // then point at q so that they are still well formed.
  const void* kp = total_k > 0 ? k : q;
  const void* vp = total_k > 0 ? v : q;
  const int krows = total_k > 0 ? total_k : total_q;
  const int kcols = total_k > 0 ? HkD : HD;
  const int kbox = head_dim == 256 ? 64 : fa::kFwdBN;  // rows per K/V tile
  if (!encode_map(&tq, q, total_q, HD, fa::kFwdBM) || !encode_map(&tk, kp, krows, kcols, kbox) ||
      !encode_map(&tv, vp, krows, kcols, kbox))
    return FA_ERR_CUDA;

  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  const long long items = static_cast<long long>(L.max_pairs) * num_heads;
  fa::FwdArgs fa_args{};
  fa_args.cu_q = cu_seqlens_q;
  fa_args.keys = keys;
  fa_args.out = out;
  fa_args.lse = softmax_lse;
  fa_args.workspace = workspace;
  fa_args.pairs_offset = L.pairs;
  fa_args.H = num_heads;
  fa_args.D = head_dim;
  fa_args.total_q = total_q;
  fa_args.group = num_heads / num_heads_k;
  fa_args.causal = causal ? 1 : 0;
  fa_args.scale_log2 = softmax_scale * 1.4426950408889634f;
  fa_args.grid = static_cast<int>(items < sms ? items : sms);
  fa_args.wait_ns = t_hooks.wait_ns;
  fa_args.withhold_v0 = head_dim == 256 ? 0 : t_hooks.withhold_v0;
  fa_args.chained = chained() ? 1 : 0;
  auto launch = head_dim == 256 ? fa::launch_fwd_d256 : fa::launch_fwd;
  if (timed_launch(stream, [&] { return launch(fa_args, tq, tk, tv, stream); }) != cudaSuccess) return FA_ERR_CUDA;
  return FA_OK;
}

// The backward; deterministic: dQ contributions added in key-tile order.
fa_status_t run_bwd(const void* dout, const void* q, const void* k, const void* v, const void* out,
                    const float* softmax_lse, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                    int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int num_heads, int num_heads_k,
                    int head_dim, float softmax_scale, int causal, void* dq, void* dk, void* dv, void* workspace,
                    size_t workspace_bytes, fa_cuda_stream_t stream_, bool deterministic) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  fa_status_t st = check_sizes(batch, total_q, total_k, max_seqlen_q, max_seqlen_k, num_heads, num_heads_k,
                               head_dim, softmax_scale);
  if (st != FA_OK) return st;
  if (!cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARGUMENT;
  if (total_q > 0 && (!q || !dout || !out || !softmax_lse || !dq || !aligned16(q) || !aligned16(dout) ||
                      !aligned16(out) || !aligned16(dq)))
    return FA_ERR_INVALID_ARGUMENT;
  if (total_k > 0 && (!k || !v || !dk || !dv || !aligned16(k) || !aligned16(v) || !aligned16(dk) || !aligned16(dv)))
    return FA_ERR_INVALID_ARGUMENT;
  const WsLayout L = fa::ws_layout(true, batch, total_q, total_k, num_heads, head_dim);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < L.total)
    return FA_ERR_WORKSPACE;

  t_events.next = 0;
  fa::SchedArgs sa{cu_seqlens_q, fa::KeyRows{cu_seqlens_k, nullptr, nullptr, 0, nullptr, 0, 0}, batch, total_q, total_k,
                   max_seqlen_q, max_seqlen_k, causal ? 1 : 0, 1, 0, deterministic ? 1 : 0, workspace, L.seq_off,
                   L.pairs, L.max_pairs};
  if (timed_launch(stream, [&] { return fa::launch_sched_prep(sa, stream); }) != cudaSuccess) return FA_ERR_CUDA;
  if (total_q == 0 && total_k == 0) return FA_OK;

  const int HD = num_heads * head_dim;
  const int HkD = num_heads_k * head_dim;
  fa::BwdMaps maps;
  const void* anyp = total_q > 0 ? q : k;
  const void* qp = total_q > 0 ? q : anyp;
  const void* dop = total_q > 0 ? dout : anyp;
  const void* kp = total_k > 0 ? k : anyp;
  const void* vp = total_k > 0 ? v : anyp;
  const int qrows = total_q > 0 ? total_q : total_k;
  const int krows = total_k > 0 ? total_k : total_q;
  // With one side empty the other side's pointer stands in; the widths then
  // follow that tensor's head count.
  const int qcols = total_q > 0 ? HD : HkD;
  const int kcols = total_k > 0 ? HkD : HD;
  // dk / dv maps serve only stores of key tiles, which exist only when total_k > 0.
  const void* dkp = total_k > 0 ? dk : anyp;
  const void* dvp = total_k > 0 ? dv : anyp;
  // head_dim 256 runs a dV pass over 128-row query tiles and a dK/dQ pass
  // over 64-row query tiles (fa_bwd_d256_sm100.cu); its dK/dV leave as rows.
  fa::BwdMapsD256 maps256;
  if (head_dim == 256) {
    if (!encode_map(&maps256.q128, qp, qrows, qcols, 128) || !encode_map(&maps256.do128, dop, qrows, qcols, 128) ||
        !encode_map(&maps256.q64, qp, qrows, qcols, 64) || !encode_map(&maps256.do64, dop, qrows, qcols, 64) ||
        !encode_map(&maps256.k, kp, krows, kcols, fa::kBwdBN) || !encode_map(&maps256.v, vp, krows, kcols, fa::kBwdBN))
      return FA_ERR_CUDA;
  } else if (!encode_map(&maps.q, qp, qrows, qcols, fa::kBwdBM) ||
             !encode_map(&maps.dout, dop, qrows, qcols, fa::kBwdBM) ||
             !encode_map(&maps.k, kp, krows, kcols, fa::kBwdBN) || !encode_map(&maps.v, vp, krows, kcols, fa::kBwdBN) ||
             !encode_map(&maps.dk, dkp, krows, kcols, fa::kBwdBN) ||
             !encode_map(&maps.dv, dvp, krows, kcols, fa::kBwdBN)) {
    return FA_ERR_CUDA;
  }
  std::memset(&maps.dqacc, 0, sizeof(maps.dqacc));
  if (head_dim == 64 && total_q > 0 &&
      !encode_map_f32(&maps.dqacc, static_cast<char*>(workspace) + L.dqacc,
                      static_cast<long long>(num_heads) * L.tq_pad, head_dim))
    return FA_ERR_CUDA;

  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  const long long items = static_cast<long long>(L.max_pairs) * num_heads_k;
  fa::BwdArgs b{};
  b.cu_q = cu_seqlens_q;
  b.keys = fa::KeyRows{cu_seqlens_k, nullptr, nullptr, 0, nullptr, 0, 0};
  b.dout = dout;
  b.out = out;
  b.lse = softmax_lse;
  b.dq = dq;
  b.dk = dk;
  b.dv = dv;
  b.workspace = workspace;
  b.pairs_offset = L.pairs;
  b.dvec_offset = L.dvec;
  b.qcount_offset = L.qcount;
  b.deterministic = deterministic ? 1 : 0;
  b.dqacc_offset = L.dqacc;
  b.tq_pad = L.tq_pad;
  b.H = num_heads;
  b.Hk = num_heads_k;
  b.group = num_heads / num_heads_k;
  b.D = head_dim;
  b.total_q = total_q;
  b.total_k = total_k;
  b.causal = causal ? 1 : 0;
  b.scale = softmax_scale;
  b.scale_log2 = softmax_scale * 1.4426950408889634f;
  b.grid = static_cast<int>(items < sms ? items : sms);
  b.wait_ns = t_hooks.wait_ns;
  b.chained = chained() ? 1 : 0;
  if (timed_launch(stream, [&] { return fa::launch_bwd_preprocess(b, stream); }) != cudaSuccess ||
      timed_launch(stream,
                   [&] {
                     return head_dim == 256 ? fa::launch_bwd_d256(b, maps256, stream)
                                            : fa::launch_bwd_main(b, maps, stream);
                   }) != cudaSuccess ||
      timed_launch(stream, [&] { return fa::launch_bwd_convert(b, stream); }) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

// Workspace of the split-KV forward: header, per-sequence offsets and the
// (sequence, token tile) list, then the split partials.
struct DecodeLayout {
  size_t seq_off, pairs, opart, lpart, total;
  int max_pairs, tq;
};
DecodeLayout decode_layout(int batch, int total_q, int H, int Hk, int D, int splits) {
  DecodeLayout L{};
  L.tq = 128 / (H / Hk);
  size_t off = sizeof(fa::WsHeader);
  L.seq_off = off;
  off = fa::align_up(off + sizeof(int32_t) * (static_cast<size_t>(batch) + 1), 256);
  L.max_pairs = fa::max_pairs(batch, total_q, L.tq);
  L.pairs = off;
  off = fa::align_up(off + 8 * static_cast<size_t>(L.max_pairs), 256);
  const size_t rows = static_cast<size_t>(total_q) * H;
  if (splits > 1) {
    L.opart = off;
    off = fa::align_up(off + sizeof(float) * splits * rows * D, 256);
    L.lpart = off;
    off = fa::align_up(off + sizeof(float) * splits * rows, 256);
  }
  L.total = off;
  return L;
}

bool kv_layout_ok(const fa_kv_layout_t* kv) {
  if (!kv || kv->total_rows < 0) return false;
  if (kv->block_table) return kv->seqlens_k && kv->page_size > 0 && kv->max_pages_per_seq > 0 && !kv->leftpad_k;
  if (kv->seqlens_k) return kv->cache_rows >= 0;
  return kv->cu_seqlens_k != nullptr;
}

}  // namespace

extern "C" {

int fa_varlen_splitkv_num_splits(int batch, int max_seqlen_q, int num_heads, int num_heads_k, int max_seqlen_k,
                                 int sm_count) {
  if (batch <= 0 || max_seqlen_q <= 0 || num_heads <= 0 || num_heads_k <= 0 || num_heads % num_heads_k != 0 ||
      max_seqlen_k <= 0)
    return 1;
  if (sm_count <= 0) sm_count = ::sm_count();
  if (sm_count <= 0) return 1;
  const int group = num_heads / num_heads_k;
  if (group > 128) return 1;
  // A query tile holds tq = floor(128 / group) tokens of one sequence (the
  // split-KV kernel's decomposition), so a sequence needs ceil(lq / tq) tiles.
  const long long tq = 128 / group;
  const long long q_tiles = (static_cast<long long>(max_seqlen_q) + tq - 1) / tq;
  const long long per_split = static_cast<long long>(batch) * num_heads_k * q_tiles;
  const int k_tiles = (max_seqlen_k + 127) / 128;
  const int max_splits = std::min(1024, std::max(1, k_tiles / 2));
  int best = 1;
  double best_fill = 0.0;
  for (int s = 1; s <= max_splits; ++s) {
    const long long units = per_split * s;
    const long long slots = (units + sm_count - 1) / sm_count * sm_count;
    const double fill = static_cast<double>(units) / static_cast<double>(slots);
    if (fill >= 0.95) {
      best = s;
      break;
    }
    if (fill > best_fill) {
      best_fill = fill;
      best = s;
    }
  }
  // Ranges of fewer than 8 key tiles are dominated by a unit's fixed costs
  // (its query tile, the pipeline fill, the partial output and its share of
  // the combine): then the smallest count whose units occupy at least 85% of
  // the SMs at once streams the cache faster, with one wave of long ranges.
  if ((k_tiles + best - 1) / best < 8)
    for (int s = 1; s < best; ++s)
      if (per_split * s * 100 >= 85LL * sm_count) return s;
  return best;
}

size_t fa_varlen_fwd_splitkv_workspace_size(int batch, int total_q, int num_heads, int num_heads_k, int head_dim,
                                            int num_splits) {
  if (batch < 1 || total_q < 0 || num_heads < 1 || num_heads_k < 1 || num_heads % num_heads_k != 0 ||
      num_heads / num_heads_k > 128 || num_splits < 1)
    return 0;
  return decode_layout(batch, total_q, num_heads, num_heads_k, head_dim, num_splits).total;
}

fa_status_t fa_varlen_fwd_splitkv(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                                  const fa_kv_layout_t* kv, int batch, int total_q, int max_seqlen_q,
                                  int max_seqlen_k, int num_heads, int num_heads_k, int head_dim, float softmax_scale,
                                  int causal, int num_splits, void* out, float* softmax_lse, void* workspace,
                                  size_t workspace_bytes, fa_cuda_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!kv_layout_ok(kv) || !cu_seqlens_q || num_splits < 1 || num_splits > 1024) return FA_ERR_INVALID_ARGUMENT;
  const int total_k = kv->total_rows;
  fa_status_t st = check_sizes(batch, total_q, total_k, max_seqlen_q, max_seqlen_k, num_heads, num_heads_k,
                               head_dim, softmax_scale);
  if (st != FA_OK) return st;
  if (head_dim == 256 || num_heads / num_heads_k > 128) return FA_ERR_UNSUPPORTED;
  if (kv->block_table && kv->page_size % fa::kFwdBN != 0) return FA_ERR_UNSUPPORTED;
  if (total_q > 0 && (!q || !out || !softmax_lse || !aligned16(q) || !aligned16(out))) return FA_ERR_INVALID_ARGUMENT;
  if (total_k > 0 && (!k || !v || !aligned16(k) || !aligned16(v))) return FA_ERR_INVALID_ARGUMENT;
  const DecodeLayout L = decode_layout(batch, total_q, num_heads, num_heads_k, head_dim, num_splits);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || workspace_bytes < L.total)
    return FA_ERR_WORKSPACE;
  const fa::KeyRows keys{kv->block_table || kv->seqlens_k ? nullptr : kv->cu_seqlens_k, kv->seqlens_k, kv->leftpad_k,
                         kv->cache_rows, kv->block_table, kv->max_pages_per_seq, kv->page_size};

  t_events.next = 0;
  // Decoding and other calls whose sequences have at most one query tile need
  // no work list: the decode kernel takes item idx as (sequence idx / (Hk *
  // splits), its only tile) and checks each sequence itself, and the call
  // only resets the header's status word and work counters.
  const bool inline_list = max_seqlen_q <= L.tq;
  if (inline_list) {
    if (cudaMemsetAsync(workspace, 0, 4 * sizeof(uint32_t), stream) != cudaSuccess) return FA_ERR_CUDA;
  } else {
    fa::SchedArgs sa{cu_seqlens_q, keys, batch, total_q, total_k, max_seqlen_q, max_seqlen_k,
                     causal ? 1 : 0, 0, L.tq, 0, workspace, L.seq_off, L.pairs, L.max_pairs};
    if (timed_launch(stream, [&] { return fa::launch_sched_prep(sa, stream); }) != cudaSuccess) return FA_ERR_CUDA;
  }
  if (total_q == 0) return FA_OK;

  const int g = num_heads / num_heads_k;
  const int HkD = num_heads_k * head_dim;
  CUtensorMap tq3, tk, tv;
  const void* kp = total_k > 0 ? k : q;
  const void* vp = total_k > 0 ? v : q;
  const int krows = total_k > 0 ? total_k : total_q;
  const int kcols = total_k > 0 ? HkD : num_heads * head_dim;
  if (!encode_map_q3(&tq3, q, total_q, num_heads, head_dim, g, L.tq) ||
      !encode_map(&tk, kp, krows, kcols, fa::kFwdBN) || !encode_map(&tv, vp, krows, kcols, fa::kFwdBN))
    return FA_ERR_CUDA;

  const int sms = sm_count();
  if (sms <= 0) return FA_ERR_CUDA;
  const long long items = static_cast<long long>(inline_list ? batch : L.max_pairs) * num_heads_k * num_splits;
  fa::DecodeArgs d{};
  d.cu_q = cu_seqlens_q;
  d.keys = keys;
  d.out = out;
  d.lse = softmax_lse;
  char* ws = static_cast<char*>(workspace);
  d.opart = num_splits > 1 ? reinterpret_cast<float*>(ws + L.opart) : nullptr;
  d.lpart = num_splits > 1 ? reinterpret_cast<float*>(ws + L.lpart) : nullptr;
  d.workspace = workspace;
  d.pairs_offset = L.pairs;
  d.H = num_heads;
  d.Hk = num_heads_k;
  d.group = g;
  d.D = head_dim;
  d.total_q = total_q;
  d.tq = L.tq;
  d.splits = num_splits;
  d.causal = causal ? 1 : 0;
  d.scale_log2 = softmax_scale * 1.4426950408889634f;
  d.grid = static_cast<int>(items < sms ? items : sms);
  d.wait_ns = t_hooks.wait_ns;
  d.inline_list = inline_list ? 1 : 0;
  d.batch = batch;
  d.total_k = total_k;
  d.max_seqlen_q = max_seqlen_q;
  d.max_seqlen_k = max_seqlen_k;
  // After the header reset the decode kernel is the call's first kernel: a
  // plain launch. The combine is chained to it.
  fa::DecodeArgs dc = d;
  d.chained = chained() && !inline_list ? 1 : 0;
  dc.chained = chained() ? 1 : 0;
  if (timed_launch(stream, [&] { return fa::launch_decode(d, tq3, tk, tv, stream); }) != cudaSuccess ||
      timed_launch(stream, [&] { return fa::launch_decode_combine(dc, stream); }) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}


size_t fa_varlen_fwd_workspace_size(int batch, int total_q, int num_heads, int head_dim) {
  if (batch < 1 || total_q < 0 || num_heads < 1) return 0;
  return fa::ws_layout(false, batch, total_q, 0, num_heads, head_dim).total;
}

size_t fa_varlen_bwd_workspace_size(int batch, int total_q, int total_k, int num_heads, int head_dim) {
  if (batch < 1 || total_q < 0 || total_k < 0 || num_heads < 1) return 0;
  return fa::ws_layout(true, batch, total_q, total_k, num_heads, head_dim).total;
}

const char* fa_status_string(fa_status_t s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARGUMENT: return "FA_ERR_INVALID_ARGUMENT";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_BAD_SEQLENS: return "FA_ERR_BAD_SEQLENS";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT";
  }
  return "FA_ERR_UNKNOWN";
}

fa_status_t fa_varlen_fwd(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                          const int32_t* cu_seqlens_k, int batch, int total_q, int total_k, int max_seqlen_q,
                          int max_seqlen_k, int num_heads, int head_dim, float softmax_scale, int causal,
                          void* out, float* softmax_lse, void* workspace, size_t workspace_bytes,
                          fa_cuda_stream_t stream) {
  return fa_varlen_fwd_gqa(q, k, v, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                           max_seqlen_k, num_heads, num_heads, head_dim, softmax_scale, causal, out, softmax_lse,
                           workspace, workspace_bytes, stream);
}

fa_status_t fa_varlen_fwd_gqa(const void* q, const void* k, const void* v, const int32_t* cu_seqlens_q,
                              const int32_t* cu_seqlens_k, int batch, int total_q, int total_k, int max_seqlen_q,
                              int max_seqlen_k, int num_heads, int num_heads_k, int head_dim, float softmax_scale,
                              int causal, void* out, float* softmax_lse, void* workspace, size_t workspace_bytes,
                              fa_cuda_stream_t stream) {
  if (!cu_seqlens_k) return FA_ERR_INVALID_ARGUMENT;
  return run_fwd(q, k, v, cu_seqlens_q, fa::KeyRows{cu_seqlens_k, nullptr, nullptr, 0, nullptr, 0, 0}, batch, total_q, total_k,
                 max_seqlen_q, max_seqlen_k, num_heads, num_heads_k, head_dim, softmax_scale, causal, out,
                 softmax_lse, workspace, workspace_bytes, stream);
}

fa_status_t fa_varlen_fwd_paged(const void* q, const void* k_pages, const void* v_pages,
                                const int32_t* cu_seqlens_q, const int32_t* seqlens_k, const int32_t* block_table,
                                int batch, int total_q, int num_pages, int page_size, int max_pages_per_seq,
                                int max_seqlen_q, int max_seqlen_k, int num_heads, int num_heads_k, int head_dim,
                                float softmax_scale, int causal, void* out, float* softmax_lse, void* workspace,
                                size_t workspace_bytes, fa_cuda_stream_t stream) {
  if (!seqlens_k || !block_table || batch < 1 || num_pages < 1 || max_pages_per_seq < 1 || page_size < 1)
    return FA_ERR_INVALID_ARGUMENT;
  if (page_size % fa::kFwdBN != 0) return FA_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(num_pages) * page_size;
  if (rows > (1ll << 31) - 1 - 2 * fa::kFwdBN ||
      static_cast<long long>(max_pages_per_seq) * page_size > (1ll << 31) - 1)
    return FA_ERR_UNSUPPORTED;
  return run_fwd(q, k_pages, v_pages, cu_seqlens_q,
                 fa::KeyRows{nullptr, seqlens_k, nullptr, 0, block_table, max_pages_per_seq, page_size}, batch,
                 total_q, static_cast<int>(rows), max_seqlen_q, max_seqlen_k, num_heads, num_heads_k, head_dim,
                 softmax_scale, causal, out, softmax_lse, workspace, workspace_bytes, stream);
}

fa_status_t fa_varlen_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* cu_seqlens_q, const int32_t* seqlens_k, const int32_t* leftpad_k,
                                  int batch, int total_q, int cache_rows, int max_seqlen_q, int num_heads,
                                  int num_heads_k, int head_dim, float softmax_scale, int causal, void* out,
                                  float* softmax_lse, void* workspace, size_t workspace_bytes,
                                  fa_cuda_stream_t stream) {
  if (!seqlens_k || batch < 1 || cache_rows < 0) return FA_ERR_INVALID_ARGUMENT;
  const long long rows = static_cast<long long>(batch) * cache_rows;
  if (rows > (1ll << 31) - 1 - 2 * fa::kFwdBN) return FA_ERR_UNSUPPORTED;
  return run_fwd(q, k_cache, v_cache, cu_seqlens_q, fa::KeyRows{nullptr, seqlens_k, leftpad_k, cache_rows, nullptr, 0, 0}, batch,
                 total_q, static_cast<int>(rows), max_seqlen_q, cache_rows, num_heads, num_heads_k, head_dim,
                 softmax_scale, causal, out, softmax_lse, workspace, workspace_bytes, stream);
}

fa_status_t fa_varlen_bwd(const void* dout, const void* q, const void* k, const void* v, const void* out,
                          const float* softmax_lse, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                          int batch, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k, int num_heads,
                          int head_dim, float softmax_scale, int causal, void* dq, void* dk, void* dv,
                          void* workspace, size_t workspace_bytes, fa_cuda_stream_t stream) {
  return fa_varlen_bwd_gqa(dout, q, k, v, out, softmax_lse, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                           max_seqlen_q, max_seqlen_k, num_heads, num_heads, head_dim, softmax_scale, causal, dq, dk,
                           dv, workspace, workspace_bytes, stream);
}

fa_status_t fa_varlen_bwd_gqa(const void* dout, const void* q, const void* k, const void* v, const void* out,
                              const float* softmax_lse, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                              int batch, int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                              int num_heads, int num_heads_k, int head_dim, float softmax_scale, int causal,
                              void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes,
                              fa_cuda_stream_t stream) {
  return run_bwd(dout, q, k, v, out, softmax_lse, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                 max_seqlen_k, num_heads, num_heads_k, head_dim, softmax_scale, causal, dq, dk, dv, workspace,
                 workspace_bytes, stream, false);
}

fa_status_t fa_varlen_bwd_deterministic(const void* dout, const void* q, const void* k, const void* v,
                                        const void* out, const float* softmax_lse, const int32_t* cu_seqlens_q,
                                        const int32_t* cu_seqlens_k, int batch, int total_q, int total_k,
                                        int max_seqlen_q, int max_seqlen_k, int num_heads, int num_heads_k,
                                        int head_dim, float softmax_scale, int causal, void* dq, void* dk, void* dv,
                                        void* workspace, size_t workspace_bytes, fa_cuda_stream_t stream) {
  return run_bwd(dout, q, k, v, out, softmax_lse, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                 max_seqlen_k, num_heads, num_heads_k, head_dim, softmax_scale, causal, dq, dk, dv, workspace,
                 workspace_bytes, stream, true);
}

void fa_set_test_hooks(uint64_t wait_limit_ns, int withhold_first_value_load) {
  t_hooks.wait_ns = wait_limit_ns ? wait_limit_ns : fa::kWaitTimeoutNs;
  t_hooks.withhold_v0 = withhold_first_value_load ? 1 : 0;
}

void fa_set_kernel_events(void* const* events, int n_pairs) {
  t_events.events = events;
  t_events.n_pairs = events ? n_pairs : 0;
  t_events.next = 0;
}

fa_status_t fa_get_device_status(const void* workspace, fa_cuda_stream_t stream_) {
  if (!workspace) return FA_ERR_INVALID_ARGUMENT;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (cudaStreamSynchronize(stream) != cudaSuccess) return FA_ERR_CUDA;
  uint32_t status = 0;
  if (cudaMemcpy(&status, workspace, sizeof status, cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  return static_cast<fa_status_t>(status);
}

}  // extern "C"
