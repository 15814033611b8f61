// C ABI of the MSA hot path: argument checks, TMA descriptors, launches.
// Declarations and the contract of every entry point are in include/msa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/msa.h"
#include "attn_decode.cuh"
#include "attn_prefill.cuh"
#include "common.cuh"
#include "index_decode.cuh"
#include "index_decode_tc.cuh"
#include "index_prefill.cuh"
#include "merge_partials.cuh"
#include "qk_rope_insert.cuh"
#include "topk.cuh"

namespace {

thread_local char g_msg[512] = "";

// optional phase events of msa_attn_prefill on this host thread (msa_set_timing_events)
thread_local cudaEvent_t g_phase_ev[4] = {nullptr, nullptr, nullptr, nullptr};
inline void phase_mark(int i, cudaStream_t stream) {
  if (g_phase_ev[i]) cudaEventRecord(g_phase_ev[i], stream);
}

msa_status_t fail(msa_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

#define CHECK_ARG(cond, ...) \
  do {                       \
    if (!(cond)) return fail(MSA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)
#define CHECK_SUP(cond, ...) \
  do {                       \
    if (!(cond)) return fail(MSA_ERR_UNSUPPORTED, __VA_ARGS__); \
  } while (0)
#define CUDA_TRY(call)                                                                         \
  do {                                                                                         \
    cudaError_t e_ = (call);                                                                   \
    if (e_ != cudaSuccess) return fail(MSA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

float softmax_scale(const msa_config_t* c) {
  return c->softmax_scale > 0.f ? c->softmax_scale : 1.0f / std::sqrt(static_cast<float>(c->head_dim));
}

msa_status_t check_config(const msa_config_t* c) {
  CHECK_ARG(c != nullptr, "cfg is NULL");
  CHECK_ARG(c->num_q_heads > 0 && c->num_kv_heads > 0 && c->idx_heads > 0 && c->topk > 0,
            "head counts and topk must be positive");
  CHECK_ARG(c->num_q_heads % c->num_kv_heads == 0, "num_q_heads must be a multiple of num_kv_heads");
  CHECK_ARG(c->idx_heads % c->num_kv_heads == 0, "idx_heads must be a multiple of num_kv_heads");
  CHECK_SUP(c->num_q_heads / c->num_kv_heads == 16, "this library needs 16 query heads per KV head");
  CHECK_SUP(c->idx_heads / c->num_kv_heads <= 4, "at most 4 indexer heads per KV group");
  CHECK_SUP(c->idx_heads <= 16, "at most 16 indexer heads");
  CHECK_SUP(c->head_dim == 128, "head_dim must be 128");
  CHECK_SUP(c->idx_dim == 64, "idx_dim must be 64");
  CHECK_SUP(c->block_size == 128, "block_size must be 128");
  CHECK_SUP(c->topk <= 64, "topk must be <= 64");
  CHECK_ARG(!(c->softmax_scale != c->softmax_scale), "softmax_scale is NaN");
  return MSA_OK;
}

msa_status_t check_batch(const msa_batch_t* b) {
  CHECK_ARG(b != nullptr, "batch is NULL");
  CHECK_ARG(b->num_seqs > 0, "num_seqs must be positive");
  CHECK_ARG(b->total_q >= 0, "total_q must be >= 0");
  CHECK_ARG(b->max_blocks_per_seq > 0, "max_blocks_per_seq must be positive");
  CHECK_SUP(b->max_blocks_per_seq <= 16384, "max_blocks_per_seq must be <= 16384");
  CHECK_ARG(b->max_q_per_seq > 0, "max_q_per_seq must be positive");
  CHECK_ARG(b->num_pages > 0, "num_pages must be positive");
  CHECK_ARG(b->q_start && b->ctx_len && b->page_table, "batch index arrays must not be NULL");
  CHECK_SUP(b->total_q < (1 << 25), "total_q must be < 2^25");
  return MSA_OK;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// tensor of `rank` dims (innermost first): bf16 with the 128-byte swizzle by default
msa_status_t make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
                      const uint32_t* box, CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                      CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t gd[5], gs[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i < rank - 1; ++i) gs[i] = strides_bytes[i];
  CUresult r = fn(m, dtype, rank, const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return MSA_OK;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

msa_status_t launched() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(MSA_ERR_CUDA, "launch failed: %s", cudaGetErrorString(e));
  return MSA_OK;
}

// ---------------------------------------------------------------- workspace plans
struct PrefillWs {
  size_t counts, offsets, tile_offsets, cursor, total_tiles, entries, tile_rec, part_lse, part_o, bytes;
  long nbuckets, max_tiles;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

PrefillWs prefill_plan(const msa_config_t* c, const msa_batch_t* b) {
  PrefillWs w{};
  w.nbuckets = static_cast<long>(b->num_seqs) * c->num_kv_heads * b->max_blocks_per_seq;
  size_t o = 0;
  auto take = [&](size_t n) { size_t at = o; o = align_up(o + n, 256); return at; };
  w.counts = take(w.nbuckets * 4);
  w.offsets = take((w.nbuckets + 1) * 4);
  w.tile_offsets = take((w.nbuckets + 1) * 4);
  w.cursor = take(w.nbuckets * 4);
  w.total_tiles = take(16);
  const size_t ent = static_cast<size_t>(b->total_q) * c->num_kv_heads * c->topk;
  w.entries = take(ent * 4);
  w.max_tiles = static_cast<long>((ent + msa::ATTP_TOK - 1) / msa::ATTP_TOK) + w.nbuckets;
  w.tile_rec = take(static_cast<size_t>(w.max_tiles) * 64);
  w.part_lse = take(static_cast<size_t>(b->total_q) * c->num_q_heads * c->topk * 4);
  w.part_o = take(static_cast<size_t>(b->total_q) * c->topk * c->num_q_heads * c->head_dim * 2);
  w.bytes = o;
  return w;
}

// Splits per (row, group) of the decode attention: a split holds at most msa::ATTD_MAXB selected
// slots, and there should be about 6 work items per SM (the persistent CTAs then finish within
// about one item of each other; 2 per SM left a quarter of the last wave idle on 64 x 128K).  The
// count is rounded so that every split holds the same number of slots (no empty trailing split).
int decode_splits(const msa_config_t* c, const msa_batch_t* b) {
  const long units = static_cast<long>(b->total_q) * c->num_kv_heads;
  const long min_split = (c->topk + msa::ATTD_MAXB - 1) / msa::ATTD_MAXB;
  if (units <= 0) return static_cast<int>(min_split);
  long want = (6L * 148 + units - 1) / units;
  want = std::max(want, min_split);
  want = std::min<long>(want, c->topk);
  const long per = (c->topk + want - 1) / want;
  return static_cast<int>((c->topk + per - 1) / per);
}

struct DecodeWs {
  size_t part_lse, part_o, items, bytes;
  int nsplit;
};

DecodeWs decode_plan(const msa_config_t* c, const msa_batch_t* b) {
  DecodeWs w{};
  w.nsplit = decode_splits(c, b);
  const size_t units = static_cast<size_t>(b->total_q) * c->num_kv_heads;
  size_t o = 0;
  auto take = [&](size_t n) { size_t at = o; o = align_up(o + n, 256); return at; };
  w.part_lse = take(units * w.nsplit * 16 * 4);
  w.part_o = take(units * w.nsplit * 16 * 128 * 4);
  w.items = take(units * w.nsplit * 6 * 16);          // one 96-byte record per work item
  w.bytes = o;
  return w;
}

__global__ void wait_forever_probe_kernel() {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    msa::mbar_init(&bar, 1);
    msa::fence_mbar_init();
    msa::mbar_wait(&bar, 0, &abort_flag);  // nothing arrives: must time out
  }
}

}  // namespace

// Tensor-core indexer (any batch shape; the streaming form is faster for few queries per sequence).
template <bool FUSED>
msa_status_t launch_index_prefill(const msa_config_t* cfg, const msa_batch_t* batch, const void* idx_q,
                                  const void* idx_k_cache, float* block_scores, int32_t* block_idx,
                                  cudaStream_t stream) {
  msa_status_t st;
  const int Hi = cfg->idx_heads, Hkv = cfg->num_kv_heads, hg = Hi / Hkv;
  const int sms = num_sms();
  CHECK_SUP(batch->num_seqs <= msa::IDXP_MAXSEQ, "at most %d sequences per tensor-core indexer call",
            msa::IDXP_MAXSEQ);
  CUtensorMap tk;
  {
    const uint64_t dims[2] = {64, static_cast<uint64_t>(batch->num_pages) * Hi * 128};
    const uint64_t strides[1] = {128};
    const uint32_t box[2] = {64, 128};
    if ((st = make_map(&tk, idx_k_cache, 2, dims, strides, box)) != MSA_OK) return st;
  }
  CUtensorMap tq;
  {
    const uint64_t dims[3] = {64, static_cast<uint64_t>(Hi), static_cast<uint64_t>(batch->total_q)};
    const uint64_t strides[2] = {128, static_cast<uint64_t>(Hi) * 128};
    const uint32_t box[3] = {64, 1, 128};
    if ((st = make_map(&tq, idx_q, 3, dims, strides, box)) != MSA_OK) return st;
  }
  msa::IdxPrefillArgs a{};
  a.scores = block_scores;
  a.block_idx = block_idx;
  a.topk = cfg->topk;
  a.q_start = batch->q_start;
  a.ctx_len = batch->ctx_len;
  a.page_table = batch->page_table;
  a.num_seqs = batch->num_seqs;
  a.total_q = batch->total_q;
  a.max_blocks = batch->max_blocks_per_seq;
  a.num_pages = batch->num_pages;
  a.Hi = Hi;
  a.Hkv = Hkv;
  a.hg = hg;
  a.block_size = cfg->block_size;
  // pieces per (query tile, group) along its key blocks, for balance over the persistent CTAs; the fused
  // form keeps each row's candidates over all of its blocks, so it takes whole tiles
  a.nsplit = FUSED ? 1 : 4;
  const int q_tile = hg * 128 * 64 * 2;
  const int xbuf = FUSED ? 128 * msa::IDXP_FUSED_SLOTS * 8 : 0;   // candidate exchange between warpgroups
  a.nqbuf = (2 * q_tile + 2 * msa::IDXP_STAGE_BYTES <= 200 * 1024 - xbuf) ? 2 : 1;
  a.stages = std::min(8, (200 * 1024 - xbuf - a.nqbuf * q_tile) / msa::IDXP_STAGE_BYTES);
  CHECK_SUP(a.stages >= 2, "indexer tiles too large for the shared-memory ring");
  const int smem = a.nqbuf * q_tile + a.stages * msa::IDXP_STAGE_BYTES + xbuf + 1024;
  CUDA_TRY(set_smem(msa::index_prefill_kernel<FUSED>, smem));
  msa::index_prefill_kernel<FUSED><<<sms, msa::IDXP_THREADS, smem, stream>>>(tq, tk, a);
  return launched();
}

extern "C" {

const char* msa_status_string(msa_status_t s) {
  switch (s) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported size or layout";
    case MSA_ERR_CUDA: return "CUDA error";
    case MSA_ERR_TIMEOUT: return "device wait timed out";
    case MSA_ERR_DEVICE_BOUNDS: return "device found an out-of-range index";
  }
  return "unknown status";
}

const char* msa_last_error(void) { return g_msg; }

int32_t msa_version(void) { return 100; }

size_t msa_prefill_workspace_bytes(const msa_config_t* cfg, const msa_batch_t* batch) {
  if (check_config(cfg) != MSA_OK || check_batch(batch) != MSA_OK) return 0;
  return prefill_plan(cfg, batch).bytes;
}

size_t msa_decode_workspace_bytes(const msa_config_t* cfg, const msa_batch_t* batch) {
  if (check_config(cfg) != MSA_OK || check_batch(batch) != MSA_OK) return 0;
  return decode_plan(cfg, batch).bytes;
}

}  // extern "C"

// The streaming (few queries per sequence) indexer over bf16 or e4m3 keys.
template <bool E4M3>
msa_status_t launch_index_decode(const msa_config_t* cfg, const msa_batch_t* batch, const void* idx_q,
                                 const void* idx_k_cache, float k_scale, float* block_scores, cudaStream_t stream) {
  msa_status_t st;
  const int Hi = cfg->idx_heads, Hkv = cfg->num_kv_heads, hg = Hi / Hkv;
  const int esz = E4M3 ? 1 : 2;
  CUtensorMap tk;
  {
    const uint64_t row = 64ull * esz;
    const uint64_t dims[4] = {64, 128, static_cast<uint64_t>(Hi), static_cast<uint64_t>(batch->num_pages)};
    const uint64_t strides[3] = {row, row * 128, static_cast<uint64_t>(Hi) * row * 128};
    const uint32_t box[4] = {64, 128, static_cast<uint32_t>(hg), 1};
    if ((st = make_map(&tk, idx_k_cache, 4, dims, strides, box,
                       E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                       E4M3 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B)) != MSA_OK)
      return st;
  }
  const int sms = num_sms();
  CHECK_SUP(batch->num_seqs <= msa::IDXD_MAXSEQ, "at most %d sequences per streaming indexer call",
            msa::IDXD_MAXSEQ);
  msa::IdxDecodeArgs a{};
  a.idx_q = static_cast<const __nv_bfloat16*>(idx_q);
  a.scores = block_scores;
  a.q_start = batch->q_start;
  a.ctx_len = batch->ctx_len;
  a.page_table = batch->page_table;
  a.num_seqs = batch->num_seqs;
  a.max_blocks = batch->max_blocks_per_seq;
  a.num_pages = batch->num_pages;
  a.Hi = Hi;
  a.Hkv = Hkv;
  a.hg = hg;
  a.block_size = cfg->block_size;
  a.stage_bytes = hg * 128 * 64 * esz;
  a.k_scale = k_scale;
  const int mq = batch->max_q_per_seq;
  if (!E4M3 && mq > 2) {
    // several queries per sequence: the tensor-core form (its shared-memory traffic does not grow with them)
    CUtensorMap tq;
    {
      const uint64_t dims[3] = {64, static_cast<uint64_t>(Hi), static_cast<uint64_t>(batch->total_q)};
      const uint64_t strides[2] = {128, static_cast<uint64_t>(Hi) * 128};
      const uint32_t box[3] = {64, 1, 16};
      if ((st = make_map(&tq, idx_q, 3, dims, strides, box)) != MSA_OK) return st;
    }
    const int q_tiles = 2 * Hi * msa::IDXT_QHEAD;
    a.stages = std::min(16, (200 * 1024 - q_tiles) / a.stage_bytes);
    CHECK_SUP(a.stages >= 2, "indexer tiles too large for the shared-memory ring");
    const int smem = a.stages * a.stage_bytes + q_tiles + 1024;
    auto go_tc = [&](auto kernel) -> msa_status_t {
      CUDA_TRY(set_smem(kernel, smem));
      kernel<<<sms, msa::IDXT_THREADS, smem, stream>>>(tk, tq, a);
      return launched();
    };
    if (mq <= 4) return go_tc(msa::index_decode_tc_kernel<4>);
    return go_tc(msa::index_decode_tc_kernel<8>);
  }
  const int nqb = mq <= 1 ? 1 : mq <= 2 ? 2 : mq <= 4 ? 4 : 8;   // compile-time query bound
  const int q_bytes = msa::idxd_groups(nqb, E4M3) * nqb * Hi * 64 * 4;   // each consumer group's queries
  a.stages = std::min(16, (msa::IDXD_SMEM_BUDGET - q_bytes) / a.stage_bytes);
  CHECK_SUP(a.stages >= 2, "indexer tiles too large for the shared-memory ring");
  const int smem = a.stages * a.stage_bytes + q_bytes + 1024;
  auto go = [&](auto kernel) -> msa_status_t {
    CUDA_TRY(set_smem(kernel, smem));
    kernel<<<sms, msa::idxd_threads(nqb, E4M3), smem, stream>>>(tk, a);
    return launched();
  };
  if (mq <= 1) return go(msa::index_decode_kernel<1, E4M3>);
  if (mq <= 2) return go(msa::index_decode_kernel<2, E4M3>);
  if (mq <= 4) return go(msa::index_decode_kernel<4, E4M3>);
  return go(msa::index_decode_kernel<8, E4M3>);
}

extern "C" {

msa_status_t msa_index_scores(const msa_config_t* cfg, const msa_batch_t* batch, const void* idx_q,
                              const void* idx_k_cache, float* block_scores, cudaStream_t stream) {
  msa_status_t st;
  if ((st = check_config(cfg)) != MSA_OK) return st;
  if ((st = check_batch(batch)) != MSA_OK) return st;
  CHECK_ARG(idx_q && idx_k_cache && block_scores, "idx_q, idx_k_cache and block_scores must not be NULL");
  CHECK_ARG(aligned16(idx_q) && aligned16(idx_k_cache) && aligned16(block_scores), "pointers must be 16-byte aligned");
  if (batch->total_q == 0) return MSA_OK;
  if (batch->max_q_per_seq <= msa::IDXD_MAXQ)
    return launch_index_decode<false>(cfg, batch, idx_q, idx_k_cache, 1.f, block_scores, stream);
  return launch_index_prefill<false>(cfg, batch, idx_q, idx_k_cache, block_scores, nullptr, stream);
}

msa_status_t msa_index_scores_fp8(const msa_config_t* cfg, const msa_batch_t* batch, const void* idx_q,
                                  const void* idx_k_cache_e4m3, float k_scale, float* block_scores,
                                  cudaStream_t stream) {
  msa_status_t st;
  if ((st = check_config(cfg)) != MSA_OK) return st;
  if ((st = check_batch(batch)) != MSA_OK) return st;
  CHECK_ARG(idx_q && idx_k_cache_e4m3 && block_scores, "idx_q, idx_k_cache_e4m3 and block_scores must not be NULL");
  CHECK_ARG(aligned16(idx_q) && aligned16(idx_k_cache_e4m3) && aligned16(block_scores),
            "pointers must be 16-byte aligned");
  CHECK_ARG(std::isfinite(k_scale) && k_scale > 0.f, "k_scale must be positive and finite");
  CHECK_SUP(batch->max_q_per_seq <= msa::IDXD_MAXQ, "the e4m3 indexer handles at most %d queries per sequence",
            msa::IDXD_MAXQ);
  if (batch->total_q == 0) return MSA_OK;
  return launch_index_decode<true>(cfg, batch, idx_q, idx_k_cache_e4m3, k_scale, block_scores, stream);
}

msa_status_t msa_topk_blocks(const msa_config_t* cfg, const msa_batch_t* batch, const float* block_scores,
                             int32_t* block_idx, cudaStream_t stream) {
  msa_status_t st;
  if ((st = check_config(cfg)) != MSA_OK) return st;
  if ((st = check_batch(batch)) != MSA_OK) return st;
  CHECK_ARG(block_scores && block_idx, "block_scores and block_idx must not be NULL");
  if (batch->total_q == 0) return MSA_OK;
  const long rows = static_cast<long>(batch->total_q) * cfg->num_kv_heads;
  const int nb = batch->max_blocks_per_seq;
  const int Hkv = cfg->num_kv_heads, k = cfg->topk, bs = cfg->block_size;
#define TOPK_ARGS block_scores, block_idx, batch->q_start, batch->ctx_len, batch->num_seqs, batch->total_q, Hkv, nb, k, bs
  if (nb <= 256) {
    msa::topk_row_warp_kernel<8><<<static_cast<unsigned>((rows + 3) / 4), 128, 0, stream>>>(TOPK_ARGS);
  } else if (nb <= 1024) {
    msa::topk_row_warp_kernel<32><<<static_cast<unsigned>((rows + 3) / 4), 128, 0, stream>>>(TOPK_ARGS);
  } else if (nb <= 2048) {
    msa::topk_blocks_kernel<2, 32><<<static_cast<unsigned>(rows), 64, 0, stream>>>(TOPK_ARGS);
  } else if (nb <= 4096) {
    msa::topk_blocks_kernel<4, 32><<<static_cast<unsigned>(rows), 128, 0, stream>>>(TOPK_ARGS);
  } else if (nb <= 8192) {
    msa::topk_blocks_kernel<8, 32><<<static_cast<unsigned>(rows), 256, 0, stream>>>(TOPK_ARGS);
  } else {
    msa::topk_blocks_kernel<16, 32><<<static_cast<unsigned>(rows), 512, 0, stream>>>(TOPK_ARGS);
  }
#undef TOPK_ARGS
  return launched();
}

msa_status_t msa_index_topk(const msa_config_t* cfg, const msa_batch_t* batch, const void* idx_q,
                            const void* idx_k_cache, int32_t* block_idx, cudaStream_t stream) {
  msa_status_t st;
  if ((st = check_config(cfg)) != MSA_OK) return st;
  if ((st = check_batch(batch)) != MSA_OK) return st;
  CHECK_ARG(idx_q && idx_k_cache && block_idx, "idx_q, idx_k_cache and block_idx must not be NULL");
  CHECK_ARG(aligned16(idx_q) && aligned16(idx_k_cache) && aligned16(block_idx), "pointers must be 16-byte aligned");
  CHECK_SUP(cfg->topk <= msa::IDXP_FUSED_SLOTS + 1, "the fused indexer keeps at most %d blocks per row",
            msa::IDXP_FUSED_SLOTS + 1);
  if (batch->total_q == 0) return MSA_OK;
  return launch_index_prefill<true>(cfg, batch, idx_q, idx_k_cache, nullptr, block_idx, stream);
}

msa_status_t msa_attn_prefill(const msa_config_t* cfg, const msa_batch_t* batch, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* block_idx, void* out, float* lse, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
  msa_status_t st;
  if ((st = check_config(cfg)) != MSA_OK) return st;
  if ((st = check_batch(batch)) != MSA_OK) return st;
  CHECK_ARG(q && k_cache && v_cache && block_idx && out, "q, caches, block_idx and out must not be NULL");
  CHECK_ARG(aligned16(q) && aligned16(k_cache) && aligned16(v_cache) && aligned16(out) && aligned16(workspace),
            "pointers must be 16-byte aligned");
  const PrefillWs w = prefill_plan(cfg, batch);
  CHECK_ARG(workspace != nullptr && workspace_bytes >= w.bytes, "workspace too small: %zu bytes needed", w.bytes);
  CHECK_SUP(w.nbuckets < (1L << 31) && w.max_tiles < (1L << 31), "too many (sequence, group, block) buckets");
  if (batch->total_q == 0) return MSA_OK;
  char* ws = static_cast<char*>(workspace);
  const int Hq = cfg->num_q_heads, Hkv = cfg->num_kv_heads, k = cfg->topk;

  msa::SchedArgs s{};
  s.block_idx = block_idx;
  s.q_start = batch->q_start;
  s.ctx_len = batch->ctx_len;
  s.counts = reinterpret_cast<int*>(ws + w.counts);
  s.offsets = reinterpret_cast<int*>(ws + w.offsets);
  s.tile_offsets = reinterpret_cast<int*>(ws + w.tile_offsets);
  s.cursor = reinterpret_cast<int*>(ws + w.cursor);
  s.entries = reinterpret_cast<int*>(ws + w.entries);
  s.total_tiles = reinterpret_cast<int*>(ws + w.total_tiles);
  s.num_seqs = batch->num_seqs;
  s.total_q = batch->total_q;
  s.Hkv = Hkv;
  s.topk = k;
  s.max_blocks = batch->max_blocks_per_seq;
  s.block_size = cfg->block_size;
  s.nbuckets = static_cast<int>(w.nbuckets);
  s.tile_rec = reinterpret_cast<int4*>(ws + w.tile_rec);
  s.page_table = batch->page_table;
  s.num_pages = batch->num_pages;
  s.max_tiles = static_cast<int>(w.max_tiles);
  phase_mark(0, stream);
  CUDA_TRY(cudaMemsetAsync(s.counts, 0, w.nbuckets * 4, stream));
  const unsigned sgrid = static_cast<unsigned>((batch->total_q + msa::SCHED_ROWS - 1) / msa::SCHED_ROWS);
  msa::sched_count_scatter_kernel<<<sgrid, 256, 0, stream>>>(s, 0);
  if ((st = launched()) != MSA_OK) return st;
  msa::sched_scan_kernel<<<1, 1024, 0, stream>>>(s);
  if ((st = launched()) != MSA_OK) return st;
  msa::sched_count_scatter_kernel<<<sgrid, 256, 0, stream>>>(s, 1);
  if ((st = launched()) != MSA_OK) return st;
  const int sms = num_sms();
  const long tgrid = std::min<long>((w.max_tiles + 255) / 256, 8L * sms);
  msa::sched_tiles_kernel<<<static_cast<unsigned>(std::max<long>(1, tgrid)), 256, 0, stream>>>(s);
  if ((st = launched()) != MSA_OK) return st;

  CUtensorMap tq, tk, tv, tpo;
  {
    const uint64_t dims[2] = {128, static_cast<uint64_t>(batch->total_q) * Hq};
    const uint64_t strides[1] = {256};
    const uint32_t box[2] = {64, 16};
    if ((st = make_map(&tq, q, 2, dims, strides, box)) != MSA_OK) return st;
  }
  {
    const uint64_t dims[2] = {128, static_cast<uint64_t>(batch->num_pages) * Hkv * 128};
    const uint64_t strides[1] = {256};
    const uint32_t box[2] = {64, 128};
    if ((st = make_map(&tk, k_cache, 2, dims, strides, box)) != MSA_OK) return st;
    if ((st = make_map(&tv, v_cache, 2, dims, strides, box)) != MSA_OK) return st;
  }
  {
    const uint64_t dims[2] = {128, static_cast<uint64_t>(batch->total_q) * k * Hq};
    const uint64_t strides[1] = {256};
    const uint32_t box[2] = {64, 16};
    if ((st = make_map(&tpo, ws + w.part_o, 2, dims, strides, box)) != MSA_OK) return st;
  }
  msa::AttnPrefillArgs a{};
  a.tile_rec = s.tile_rec;
  a.total_tiles = s.total_tiles;
  a.part_lse = reinterpret_cast<float*>(ws + w.part_lse);
  a.Hq = Hq;
  a.topk = k;
  a.max_tiles = s.max_tiles;
  a.scale_log2 = softmax_scale(cfg) * 1.4426950408889634f;
  CUDA_TRY(set_smem(msa::attn_prefill_kernel, msa::ATTP_SMEM));
  phase_mark(1, stream);
  msa::attn_prefill_kernel<<<sms, msa::ATTP_THREADS, msa::ATTP_SMEM, stream>>>(tq, tk, tv, tpo, a);
  if ((st = launched()) != MSA_OK) return st;
  phase_mark(2, stream);

  msa::MergeArgs m{};
  m.part_o = reinterpret_cast<const __nv_bfloat16*>(ws + w.part_o);
  m.part_lse = a.part_lse;
  m.block_idx = block_idx;
  m.out = static_cast<__nv_bfloat16*>(out);
  m.lse = lse;
  m.total_q = batch->total_q;
  m.Hq = Hq;
  m.Hkv = Hkv;
  m.topk = k;
  msa::attn_merge_kernel<<<static_cast<unsigned>(batch->total_q) * Hkv, 256, 0, stream>>>(m);
  if ((st = launched()) != MSA_OK) return st;
  phase_mark(3, stream);
  return MSA_OK;
}

msa_status_t msa_set_timing_events(void* const* events, int32_t n) {
  CHECK_ARG(n == 0 || (n == 4 && events != nullptr), "pass 4 events, or 0 to stop recording");
  for (int i = 0; i < 4; ++i) g_phase_ev[i] = n ? static_cast<cudaEvent_t>(events[i]) : nullptr;
  return MSA_OK;
}

msa_status_t msa_attn_decode(const msa_config_t* cfg, const msa_batch_t* batch, const void* q, const void* k_cache,
                             const void* v_cache, const int32_t* block_idx, void* out, float* lse, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  msa_status_t st;
  if ((st = check_config(cfg)) != MSA_OK) return st;
  if ((st = check_batch(batch)) != MSA_OK) return st;
  CHECK_ARG(q && k_cache && v_cache && block_idx && out, "q, caches, block_idx and out must not be NULL");
  CHECK_ARG(aligned16(q) && aligned16(k_cache) && aligned16(v_cache) && aligned16(out) && aligned16(workspace),
            "pointers must be 16-byte aligned");
  const DecodeWs w = decode_plan(cfg, batch);
  CHECK_ARG(workspace != nullptr && workspace_bytes >= w.bytes, "workspace too small: %zu bytes needed", w.bytes);
  if (batch->total_q == 0) return MSA_OK;
  char* ws = static_cast<char*>(workspace);
  msa::AttnDecodeArgs a{};
  a.block_idx = block_idx;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.q_start = batch->q_start;
  a.ctx_len = batch->ctx_len;
  a.page_table = batch->page_table;
  a.part_o = reinterpret_cast<float*>(ws + w.part_o);
  a.part_lse = reinterpret_cast<float*>(ws + w.part_lse);
  a.items = reinterpret_cast<int4*>(ws + w.items);
  a.num_seqs = batch->num_seqs;
  a.total_q = batch->total_q;
  a.Hq = cfg->num_q_heads;
  a.Hkv = cfg->num_kv_heads;
  a.topk = cfg->topk;
  a.max_blocks = batch->max_blocks_per_seq;
  a.num_pages = batch->num_pages;
  a.block_size = cfg->block_size;
  a.nsplit = w.nsplit;
  a.scale_log2 = softmax_scale(cfg) * 1.4426950408889634f;
  const size_t units = static_cast<size_t>(batch->total_q) * cfg->num_kv_heads;
  CHECK_SUP(units * w.nsplit < (size_t(1) << 31), "too many (row, group, split) work items");
  a.per = (cfg->topk + w.nsplit - 1) / w.nsplit;
  a.n_items = static_cast<int>(units * w.nsplit);
  CUtensorMap tq, tk, tv;
  {
    const uint64_t dims[2] = {128, static_cast<uint64_t>(batch->total_q) * cfg->num_q_heads};
    const uint64_t strides[1] = {256};
    const uint32_t box[2] = {64, 16};
    if ((st = make_map(&tq, q, 2, dims, strides, box)) != MSA_OK) return st;
  }
  {
    const uint64_t dims[2] = {128, static_cast<uint64_t>(batch->num_pages) * cfg->num_kv_heads * 128};
    const uint64_t strides[1] = {256};
    const uint32_t box[2] = {64, 128};
    if ((st = make_map(&tk, k_cache, 2, dims, strides, box)) != MSA_OK) return st;
    if ((st = make_map(&tv, v_cache, 2, dims, strides, box)) != MSA_OK) return st;
  }
  msa::attn_decode_plan_kernel<<<static_cast<unsigned>((a.n_items + 255) / 256), 256, 0, stream>>>(a);
  if ((st = launched()) != MSA_OK) return st;
  CUDA_TRY(set_smem(msa::attn_decode_kernel, msa::ATTD_SMEM));
  const int grid = static_cast<int>(std::min<long>(a.n_items, num_sms()));
  msa::attn_decode_kernel<<<grid, msa::ATTD_THREADS, msa::ATTD_SMEM, stream>>>(tq, tk, tv, a);
  if ((st = launched()) != MSA_OK) return st;
  if (w.nsplit > 1) {
    msa::attn_decode_merge_kernel<<<static_cast<unsigned>(units), 256, 0, stream>>>(a);
    if ((st = launched()) != MSA_OK) return st;
  }
  return MSA_OK;
}

msa_status_t msa_qknorm_rope_insert(const msa_config_t* cfg, const msa_batch_t* batch, void* q, const void* k_new,
                                    const void* v_new, const void* q_norm_w, const void* k_norm_w, void* k_cache,
                                    void* v_cache, int32_t rotary_dim, float rope_theta, float eps,
                                    cudaStream_t stream) {
  msa_status_t st;
  if ((st = check_config(cfg)) != MSA_OK) return st;
  if ((st = check_batch(batch)) != MSA_OK) return st;
  CHECK_ARG(q && k_new && v_new && q_norm_w && k_norm_w && k_cache && v_cache,
            "q, k_new, v_new, the norm weights and the caches must not be NULL");
  CHECK_ARG(aligned16(q) && aligned16(k_new) && aligned16(v_new) && aligned16(q_norm_w) && aligned16(k_norm_w) &&
                aligned16(k_cache) && aligned16(v_cache),
            "pointers must be 16-byte aligned");
  CHECK_ARG(rotary_dim > 0 && rotary_dim % 8 == 0 && rotary_dim <= cfg->head_dim,
            "rotary_dim must be a positive multiple of 8, at most head_dim");
  CHECK_ARG(std::isfinite(rope_theta) && rope_theta > 0.f, "rope_theta must be positive and finite");
  CHECK_ARG(std::isfinite(eps) && eps >= 0.f, "eps must be finite and >= 0");
  if (batch->total_q == 0) return MSA_OK;
  msa::QkRopeArgs a{};
  a.q = static_cast<__nv_bfloat16*>(q);
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.q_w = static_cast<const __nv_bfloat16*>(q_norm_w);
  a.k_w = static_cast<const __nv_bfloat16*>(k_norm_w);
  a.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  a.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  a.q_start = batch->q_start;
  a.ctx_len = batch->ctx_len;
  a.page_table = batch->page_table;
  a.num_seqs = batch->num_seqs;
  a.total_q = batch->total_q;
  a.Hq = cfg->num_q_heads;
  a.Hkv = cfg->num_kv_heads;
  a.max_blocks = batch->max_blocks_per_seq;
  a.num_pages = batch->num_pages;
  a.block_size = cfg->block_size;
  a.rotary_dim = rotary_dim;
  a.log2_theta = std::log2(static_cast<double>(rope_theta));
  a.eps = eps;
  const int smem = msa::qkr_smem_bytes(a.Hq, a.Hkv);
  CUDA_TRY(set_smem(msa::qk_rope_insert_kernel, smem));
  // eight CTAs per SM need their shared memory more than L1 (no data is reused)
  CUDA_TRY(cudaFuncSetAttribute(msa::qk_rope_insert_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared));
  msa::qk_rope_insert_kernel<<<static_cast<unsigned>(batch->total_q), msa::QKR_THREADS, smem, stream>>>(a);
  return launched();
}

msa_status_t msa_merge_partials(int32_t n, int64_t units, int32_t head_dim, const void* outs, const float* lses,
                                void* out, float* lse, cudaStream_t stream) {
  CHECK_ARG(n >= 1 && n <= 4096, "n must be in [1, 4096]");
  CHECK_ARG(units >= 0, "units must be >= 0");
  CHECK_SUP(head_dim == 128, "head_dim must be 128");
  CHECK_ARG(outs && lses && out, "outs, lses and out must not be NULL");
  CHECK_ARG(aligned16(outs) && aligned16(out) && (reinterpret_cast<uintptr_t>(lses) & 3u) == 0 &&
                (reinterpret_cast<uintptr_t>(lse) & 3u) == 0,
            "outs and out must be 16-byte aligned, lses and lse 4-byte aligned");
  if (units == 0) return MSA_OK;
  const long warps_per_cta = msa::MRG_THREADS / 32;
  const long grid = (units + warps_per_cta - 1) / warps_per_cta;
  CHECK_SUP(grid <= 0x7FFFFFFFL, "too many rows");
  msa::merge_partials_kernel<<<static_cast<unsigned>(grid), msa::MRG_THREADS, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(outs), lses, static_cast<__nv_bfloat16*>(out), lse, n, units);
  return launched();
}

msa_status_t msa_get_device_status(cudaStream_t stream) {
  CUDA_TRY(cudaStreamSynchronize(stream));
  unsigned int word = 0, zero = 0;
  CUDA_TRY(cudaMemcpyFromSymbol(&word, msa::g_error, sizeof(word)));
  CUDA_TRY(cudaMemcpyToSymbol(msa::g_error, &zero, sizeof(zero)));
  if (word & msa::MSA_DEV_TIMEOUT) return fail(MSA_ERR_TIMEOUT, "a device-side wait timed out");
  if (word & msa::MSA_DEV_BOUNDS) return fail(MSA_ERR_DEVICE_BOUNDS, "the device found an out-of-range index");
  return MSA_OK;
}

msa_status_t msa_set_wait_limit_ns(uint64_t ns) {
  CHECK_ARG(ns > 0, "the wait limit must be positive");
  unsigned long long v = ns;
  CUDA_TRY(cudaMemcpyToSymbol(msa::g_wait_limit_ns, &v, sizeof(v)));
  return MSA_OK;
}

msa_status_t msa_debug_wait_timeout(cudaStream_t stream) {
  wait_forever_probe_kernel<<<1, 32, 0, stream>>>();
  return launched();
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free decode attention
// Some callers cannot hand this library a workspace: a plugin driven by a host
// framework that passes it only input and output buffers has no allocator of
// its own, and a serving loop may forbid cudaMalloc on the per-step path
// (it can synchronize the device and its latency is unbounded).  For them
// msa_attn_decode_noalloc keeps the split partials and work-item records of the
// decode attention in this fixed device array instead.  The array is part of
// the library's device code: every GPU that loads the library holds it until
// the process exits.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kNoAllocMaxDevices = 64;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};

// Device address of the array on the current device.  In host code the name
// g_noalloc_scratch only stands for the symbol; the first call on each device
// asks the runtime for the real address (cudaGetSymbolAddress) and keeps it.
// The address belongs to the current device, so `stream` must belong to it too.
msa_status_t noalloc_scratch(cudaStream_t stream, void** out) {
  int dev = -1;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(MSA_ERR_UNSUPPORTED, "device %d out of range", dev);
  int sdev = dev;
  CUDA_TRY(cudaStreamGetDevice(stream, &sdev));
  if (sdev != dev)
    return fail(MSA_ERR_INVALID_ARG, "the stream belongs to device %d but device %d is current", sdev, dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return MSA_OK;
}
}  // namespace

extern "C" msa_status_t msa_attn_decode_noalloc(const msa_config_t* cfg, const msa_batch_t* batch, const void* q,
                                                const void* k_cache, const void* v_cache, const int32_t* block_idx,
                                                void* out, float* lse, cudaStream_t stream) {
  msa_status_t st;
  if ((st = check_config(cfg)) != MSA_OK) return st;
  if ((st = check_batch(batch)) != MSA_OK) return st;
  const size_t need = decode_plan(cfg, batch).bytes;
  if (need > kNoAllocScratchBytes)
    return fail(MSA_ERR_UNSUPPORTED,
                "this batch needs %zu bytes of decode scratch, more than the %zu-byte static area of "
                "msa_attn_decode_noalloc; split the batch or use msa_attn_decode with a workspace",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if ((st = noalloc_scratch(stream, &scratch)) != MSA_OK) return st;
  return msa_attn_decode(cfg, batch, q, k_cache, v_cache, block_idx, out, lse, scratch, kNoAllocScratchBytes,
                         stream);
}

