/*
 * msa.h - C ABI of the MiniMax Sparse Attention (MSA) hot path for B200 (sm_100a).
 *
 * The method (sources: "MiniMax M3: 1M-token multimodal reasoning model now
 * available with NVIDIA and vLLM support", daily.dev, sections "Summary" and
 * "What makes M3 different"; "MiniMax-M3", inteligile model page, table
 * "Checked in its code"; "MiniMax M3 in vLLM: Day-0-Unterstuetzung ...",
 * 24-ai.news; "Serving AI agents at scale ...", shaam.blog, section "What
 * makes MiniMax M3 different from other open-weight models?"):
 * the KV sequence is cut into 128-token blocks; a lightweight indexer scores
 * every causally visible block for each query and GQA group; the top-k blocks
 * are kept; GQA attention (64 query heads over 4 KV heads) runs only over the
 * kept, uncompressed blocks.
 *
 * Readings this library fixes where the pages are silent: block score = sum
 * over the group's indexer heads of the max over the block's visible keys of
 * the raw dot product; the query's own block is always kept; ties go to the
 * lower block id; softmax scale 1/sqrt(head_dim) unless given.
 *
 * CONVENTIONS (all entry points)
 *   - Every pointer argument except `cfg`/`batch` themselves and the host
 *     fields of msa_batch_t is a DEVICE pointer on the current CUDA device.
 *   - The caller owns all memory.  No entry point allocates device memory;
 *     scratch space is passed in as `workspace`.
 *   - Work is enqueued on `stream`; nothing synchronises the host except
 *     msa_get_device_status().
 *   - Arguments are checked before anything is launched; a failed check
 *     returns MSA_ERR_INVALID_ARG / MSA_ERR_UNSUPPORTED and launches nothing
 *     (msa_last_error() tells why).  A failed launch returns MSA_ERR_CUDA.
 *   - Index errors found on the device (page id outside [0, num_pages), a
 *     selected block after the query's block, more queries per sequence than
 *     declared) and bounded waits that ran out are recorded in a device error
 *     word and reported by msa_get_device_status(); the kernels skip the bad
 *     access instead of faulting.
 *   - Cache slots of a page past a sequence's ctx_len (the unwritten tail of
 *     its last page) must hold finite values: the tensor-core P.V multiplies
 *     those V rows by zero probabilities, and 0 * NaN is NaN.  Pages that come
 *     zeroed or hold earlier finite writes satisfy this.
 *
 * LAYOUTS (row-major, bf16 = IEEE bfloat16, fp32 = IEEE float)
 *   idx_q        bf16 [total_q][idx_heads][idx_dim]
 *   idx_k_cache  bf16 [num_pages][idx_heads][block_size][idx_dim]
 *   q            bf16 [total_q][num_q_heads][head_dim]
 *   k_cache      bf16 [num_pages][num_kv_heads][block_size][head_dim]   (v_cache alike)
 *   block_scores fp32 [total_q][num_kv_heads][max_blocks_per_seq]
 *   block_idx    int32 [total_q][num_kv_heads][topk]   ascending ids, -1 padded
 *   out          bf16 [total_q][num_q_heads][head_dim]
 *   lse          fp32 [total_q][num_q_heads]  (natural log; may be NULL)
 *   Query row t belongs to sequence s with q_start[s] <= t < q_start[s+1];
 *   its position is p = ctx_len[s] - (q_start[s+1] - q_start[s]) + (t - q_start[s]),
 *   i.e. the call's queries are the last tokens of the context, whose keys
 *   are already in the caches.  Key block b of sequence s lives in physical
 *   page page_table[s][b].  A prefill is the same call with an identity
 *   page table.
 *
 * Supported sizes: head_dim 128, idx_dim 64, block_size 128,
 * num_q_heads = 16 * num_kv_heads, idx_heads a multiple of num_kv_heads with
 * at most 4 indexer heads per group, 1 <= topk <= 64, max_blocks_per_seq <=
 * 16384 (2M tokens).  Pointers must be 16-byte aligned.
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,  /* a pointer, size or layout argument is wrong        */
  MSA_ERR_UNSUPPORTED = 2,  /* valid, but outside the sizes this library handles  */
  MSA_ERR_CUDA = 3,         /* a CUDA runtime / driver call failed                 */
  MSA_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out (status query)   */
  MSA_ERR_DEVICE_BOUNDS = 5 /* the device found an out-of-range index (status)     */
} msa_status_t;

typedef struct {
  int32_t num_q_heads;   /* H_q  (64 in the pages' configuration)                  */
  int32_t num_kv_heads;  /* H_kv (4); H_q / H_kv query heads share one KV head      */
  int32_t head_dim;      /* 128                                                     */
  int32_t idx_heads;     /* indexer heads H_i, split contiguously over the KV groups */
  int32_t idx_dim;       /* indexer head dim, 64                                    */
  int32_t block_size;    /* tokens per KV block = tokens per cache page, 128        */
  int32_t topk;          /* blocks kept per (query, group), current block included   */
  float softmax_scale;   /* <= 0 selects 1 / sqrt(head_dim)                          */
} msa_config_t;

typedef struct {
  int32_t num_seqs;           /* host: sequences in the batch                       */
  int32_t total_q;            /* host: query rows in the call = q_start[num_seqs]   */
  int32_t max_blocks_per_seq; /* host: row width of page_table and block_scores      */
  int32_t max_q_per_seq;      /* host: upper bound of any sequence's query count     */
  int32_t num_pages;          /* host: pages in every cache (page ids are < this)    */
  const int32_t* q_start;     /* device [num_seqs + 1], q_start[0] = 0, non-decreasing */
  const int32_t* ctx_len;     /* device [num_seqs], context length incl. this call's queries */
  const int32_t* page_table;  /* device [num_seqs][max_blocks_per_seq]               */
} msa_batch_t;

/*
 * Indexer block scores.  For query row t (position p), KV group g and block
 * b <= p / block_size:
 *   block_scores[t][g][b] = sum_{h in heads(g)} max_{j in b, j <= p} idx_q[t][h] . idx_k[j][h]
 * with heads(g) = {g*H_i/H_kv, ..., (g+1)*H_i/H_kv - 1}, accumulated in fp32
 * from bf16 products.  Entries b > p / block_size are left undefined (the
 * call may write -inf there or leave them untouched).
 * (inteligile "MiniMax-M3", row "Indexer-selected sparse attention":
 * per-head key scores pooled into blocks; 24-ai.news: every query or GQA
 * query group scores all available blocks with lightweight indexer kernels.)
 * Calls with max_q_per_seq <= 8 stream the pages (decode / verify); larger
 * ones run the tensor-core form.
 */
msa_status_t msa_index_scores(const msa_config_t* cfg, const msa_batch_t* batch, const void* idx_q,
                              const void* idx_k_cache, float* block_scores, cudaStream_t stream);

/*
 * msa_index_scores over an FP8 indexer-key cache, for calls with at most 8
 * queries per sequence (decode and verify; MSA_ERR_UNSUPPORTED otherwise).
 * The pages list "FP8 KV-cache paths" among the upcoming work (daily.dev
 * "MiniMax M3 ...", section "What's coming") and fix no format; this library
 * reads e4m3 ("fn": finite range +-448, subnormals down to 2^-9) codes with
 * one float scale for the whole cache:
 *   idx_k_cache_e4m3  uint8 [num_pages][idx_heads][block_size][idx_dim], the
 *                     e4m3 bit patterns; key value = code * k_scale
 * (a writer stores e4m3(clamp(x / k_scale, -448, 448)), rounded to nearest
 * even).  block_scores are those of msa_index_scores on the read-back keys:
 *   block_scores[t][g][b] = sum_{h in heads(g)} max_{j in b, j <= p} idx_q[t][h] . (code[j][h] * k_scale)
 * computed as k_scale times the fp32 dot products of the bf16 queries with the
 * codes widened exactly.  k_scale must be positive and finite
 * (MSA_ERR_INVALID_ARG otherwise).  Everything else as msa_index_scores.
 */
msa_status_t msa_index_scores_fp8(const msa_config_t* cfg, const msa_batch_t* batch, const void* idx_q,
                                  const void* idx_k_cache_e4m3, float k_scale, float* block_scores,
                                  cudaStream_t stream);

/*
 * Top-k block selection per (query row, group).  cur = p / block_size is
 * always kept; the other topk-1 slots take the best blocks b < cur with a
 * finite score, ranked by (score descending, b ascending); a -inf score is
 * never kept.  Written ascending and padded with -1 to topk entries.
 * (inteligile "MiniMax-M3", row "Indexer-selected sparse attention":
 * k = min(topk_blocks, #blocks), -inf-scored slots reported as -1.)
 * Reads block_scores[t][g][0 .. cur-1] only.  Deterministic.
 */
msa_status_t msa_topk_blocks(const msa_config_t* cfg, const msa_batch_t* batch, const float* block_scores,
                             int32_t* block_idx, cudaStream_t stream);

/*
 * msa_index_scores followed by msa_topk_blocks in one pass, without the score
 * matrix: while a row's key blocks stream through the tensor-core indexer, its
 * best topk-1 earlier blocks are kept on chip by the same (score desc, block
 * asc) rule, from the same fp32 scores, so block_idx is identical to the
 * two-call result.  (24-ai.news: each query group scores all blocks with
 * light indexer score kernels and keeps only the most relevant; inteligile
 * "MiniMax-M3" model page, tag "Exp-free TopK kernel".  The pages do not say
 * whether the two are fused; this call is this library's fused form.)
 * block_idx: int32 [total_q][num_kv_heads][topk].
 * Requires topk <= 16 (MSA_ERR_UNSUPPORTED otherwise).  Always runs the
 * tensor-core form; batches with few queries per sequence are better served
 * by the two calls.
 */
msa_status_t msa_index_topk(const msa_config_t* cfg, const msa_batch_t* batch, const void* idx_q,
                            const void* idx_k_cache, int32_t* block_idx, cudaStream_t stream);

/*
 * Sparse GQA attention, block-major ("KV outer, gather Q": shaam.blog,
 * section "What makes MiniMax M3 different ..."; daily.dev, "Serving
 * options": KV-block-major prefill scheduling).  Query head h of row t uses
 * KV head g = h / (H_q / H_kv) and the keys j <= p of the blocks in
 * block_idx[t][g][:]:
 *   out[t][h] = sum_j softmax_j(scale * q[t][h] . k[j][g]) v[j][g],
 *   lse[t][h] = log sum_j exp(scale * q[t][h] . k[j][g])
 * (plain softmax, no sink, no output gate: inteligile rows "Grouped-query
 * attention", "Learnable attention sink", "Gated attention output").
 * Each selected block is loaded once per CTA run; per-(row, head, slot)
 * partial results go to `workspace` and are merged by log-sum-exp.
 * `workspace` must hold msa_prefill_workspace_bytes(cfg, batch) bytes.
 */
msa_status_t msa_attn_prefill(const msa_config_t* cfg, const msa_batch_t* batch, const void* q,
                              const void* k_cache, const void* v_cache, const int32_t* block_idx, void* out,
                              float* lse, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Same result as msa_attn_prefill, organised for few queries per sequence:
 * the selected slots of each (row, group) are split into runs of at most 8
 * blocks, each run's blocks go through the tensor cores in swap-AB form and
 * are combined by log-sum-exp, then a second kernel merges the runs the same
 * way.  `workspace` must hold msa_decode_workspace_bytes(cfg, batch) bytes;
 * nothing in it needs to be initialised.
 */
msa_status_t msa_attn_decode(const msa_config_t* cfg, const msa_batch_t* batch, const void* q,
                             const void* k_cache, const void* v_cache, const int32_t* block_idx, void* out,
                             float* lse, void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Same result as msa_attn_decode, for callers that cannot provide a workspace:
 * a plugin that a host framework hands only its input and output buffers has
 * no allocator to get one from, and some serving loops must not call
 * cudaMalloc per step (it may synchronize the device and takes unbounded
 * time).  The scratch lives in a fixed 16 MiB device array inside the library
 * (held by every GPU that loads it until exit); this call allocates nothing.
 * The pages describing MSA have no counterpart of this call.
 *   - Batches whose decode scratch (msa_decode_workspace_bytes) exceeds 16 MiB
 *     are rejected with MSA_ERR_UNSUPPORTED and a message; nothing is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) and remembers it; make that first call before any
 *     stream capture.  The remembered address dies with the device's primary
 *     context: do not call this entry point again in a process that has reset
 *     the device (cudaDeviceReset).
 *   - `stream` must belong to the current device (MSA_ERR_INVALID_ARG
 *     otherwise), whose copy of the array the call uses.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents; nothing in it needs to start at zero (every call writes what
 *     it reads).  Calls that can overlap on the GPU (different streams, or
 *     concurrent host threads) race on the array: serialize them.
 */
msa_status_t msa_attn_decode_noalloc(const msa_config_t* cfg, const msa_batch_t* batch, const void* q,
                                     const void* k_cache, const void* v_cache, const int32_t* block_idx, void* out,
                                     float* lse, cudaStream_t stream);

/*
 * The step just before the path, fused: per-head QK normalization, partial
 * rotary embedding and the paged K/V insert of this call's new rows
 * ("MiniMax-M3", inteligile model page, table "Checked in its code", rows
 * "QK normalization" and "Partial RoPE"; daily.dev "MiniMax M3 ...", section
 * "Serving options": fused QKNorm + RoPE + KV insert).  For every new row t of
 * sequence s at absolute position p = ctx_len[s] - n_q(s) + i (the i-th of the
 * sequence's n_q new rows):
 *   q[t][h]                                 = rope(rmsnorm(q[t][h]) * q_norm_w)   (in place)
 *   k_cache[page][g][p % block_size][:]     = rope(rmsnorm(k_new[t][g]) * k_norm_w)
 *   v_cache[page][g][p % block_size][:]     = v_new[t][g],   page = page_table[s][p / block_size]
 * rmsnorm(x) = x / sqrt(mean over the head's head_dim channels of x^2 + eps);
 * rope turns channel pairs (i, i + rotary_dim/2), i < rotary_dim/2, by the
 * angle p * rope_theta^(-2i / rotary_dim) (first of the pair: a cos - b sin,
 * second: b cos + a sin); channels from rotary_dim on pass through.  The pages
 * fix rotary_dim = 64 of 128; they give neither rope_theta nor eps, so both are
 * arguments.  Angles are formed in double precision.
 *   q         bf16 [total_q][num_q_heads][head_dim], read and overwritten
 *   k_new     bf16 [total_q][num_kv_heads][head_dim]   (v_new alike)
 *   q_norm_w  bf16 [head_dim], shared by the query heads (k_norm_w: key heads)
 *   k_cache   bf16 [num_pages][num_kv_heads][block_size][head_dim] (v_cache alike)
 * rotary_dim must be a positive multiple of 8, at most head_dim.  A page id
 * outside [0, num_pages) is recorded as MSA_ERR_DEVICE_BOUNDS and that row's
 * cache writes are skipped (its queries are still written).  k_new and v_new
 * must not overlap the caches or q.
 */
msa_status_t msa_qknorm_rope_insert(const msa_config_t* cfg, const msa_batch_t* batch, void* q, const void* k_new,
                                    const void* v_new, const void* q_norm_w, const void* k_norm_w, void* k_cache,
                                    void* v_cache, int32_t rotary_dim, float rope_theta, float eps,
                                    cudaStream_t stream);

/*
 * Log-sum-exp merge of n partial attentions over disjoint key sets ("LSE
 * fusion", "Two-phase forward": inteligile "MiniMax-M3" model page, tags), as
 * needed to join the results of one sequence whose KV blocks sit on several
 * GPUs:  L = log sum_s exp(lse_s),  out = sum_s exp(lse_s - L) out_s.
 *   outs  bf16 [n][units][head_dim]   each partial normalised over its own keys
 *   lses  fp32 [n][units]             natural log; -inf = the partial saw no key (weight 0)
 *   out   bf16 [units][head_dim]      lse fp32 [units] (L), or NULL
 * units = rows x heads; head_dim must be 128.  Rows whose partials are all
 * -inf get out = 0 and lse = -inf.
 */
msa_status_t msa_merge_partials(int32_t n, int64_t units, int32_t head_dim, const void* outs, const float* lses,
                                void* out, float* lse, cudaStream_t stream);

/* Timing hook (no counterpart on the pages).  With n = 4 and four cudaEvent_t
 * handles (owned by the caller), every later msa_attn_prefill call on this host
 * thread records events[0] before its schedule kernels, events[1] before the
 * block-major attention kernel, events[2] after it and events[3] after the
 * merge, on its stream, so the phases can be timed with cudaEventElapsedTime.
 * n = 0 stops recording.  Any other n is MSA_ERR_INVALID_ARG. */
msa_status_t msa_set_timing_events(void* const* events, int32_t n);

/* Workspace sizes (bytes) for the two attention calls; only the host fields of
 * `batch` are read.  0 means the arguments are invalid. */
size_t msa_prefill_workspace_bytes(const msa_config_t* cfg, const msa_batch_t* batch);
size_t msa_decode_workspace_bytes(const msa_config_t* cfg, const msa_batch_t* batch);

/* Synchronises `stream`, then reads and clears the current device's error
 * word: MSA_OK, MSA_ERR_TIMEOUT or MSA_ERR_DEVICE_BOUNDS (MSA_ERR_CUDA if the
 * stream itself reports an error). */
msa_status_t msa_get_device_status(cudaStream_t stream);

/* Sets the wall-clock limit of every device-side wait on the current device
 * (default 2 s); used by tests of the timeout path.  0 is rejected. */
msa_status_t msa_set_wait_limit_ns(uint64_t ns);

/* Test hook for the timeout path: launches one CTA that waits on an mbarrier
 * nothing will ever complete; it must give up after the wait limit, record
 * MSA_ERR_TIMEOUT and exit.  Never faults. */
msa_status_t msa_debug_wait_timeout(cudaStream_t stream);

const char* msa_status_string(msa_status_t status);
/* Message of the last failed call on this host thread ("" if none). */
const char* msa_last_error(void);
/* ABI version: major * 10000 + minor * 100 + patch. */
int32_t msa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
