/*
 * msa.h — C ABI of libmsa.so: MiniMax-Sparse-Attention (MSA) decode over an
 * NVFP4 KV cache, hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * The method (source: "vLLM Adds Day-0 Support for MiniMax-M3.1-Flash on
 * NVIDIA and AMD GPUs", ainewsbites.com, section "A model built for efficient
 * inference"): the KV cache is cut into blocks of 128 tokens; a lightweight
 * indexer scores every key of the context and the scores are pooled into one
 * score per block; exact attention then runs over the top 16 blocks only,
 * the most recent block always kept, so a query sees at most 2,048 keys.
 * Keys, values and indexer keys are stored as NVFP4 ("vLLM delivers day-0
 * support for MiniMax-M3.1-Flash", readmex.ai, TL;DR).
 *
 * Readings this library fixes where the pages are silent:
 *   indexer   s_j = sum_h w_h * max(0, q_idx[h] . k_idx[j]); one index key per
 *             token, shared by the HI indexer heads; w_h = 1 when w_idx = NULL.
 *   pooling   mean (pool_mode 0) or max (pool_mode 1) of s_j over the block's
 *             visible tokens; a block with no visible token scores -inf.
 *   selection the query's own block r = pos div 128, plus the best
 *             min(15, r) other blocks by (score desc, block index asc);
 *             written ascending, padded with -1 to 16 entries.
 *   attention o = softmax(scale * q.K^T) V over the selected keys j <= pos;
 *             query head h reads KV head h / (Hq / Hkv).
 *   positions sequence b holds L_b = seq_lens[b] tokens, its Tq query tokens
 *             last; query t sits at pos = L_b - Tq + t and sees keys 0..pos.
 *
 * NVFP4 layout (one cache = two planes + one fp32):
 *   data  [B][heads][lmax][dim/2]  uint8, E2M1 codes, element 2i in the low
 *                                   nibble of byte i, element 2i+1 in the high;
 *   scale [B][heads][lmax][dim/16] uint8, E4M3 (OCP "FN", bias 7, max 448),
 *                                   one per 16 consecutive elements;
 *   tensor_scale                    fp32 > 0, one per cache tensor.
 *   value = fp32(e2m1 * e4m3) * tensor_scale.   9/16 byte per element.
 *
 * Interface notes: the device status word is a field of msa_params_t (every
 * kernel reports through it), msa_decode also returns the log-sum-exp, and
 * msa_attend needs no scratch (its split over the selected blocks is merged on
 * chip).
 *
 * Conventions for every entry point:
 *   - pointers are DEVICE pointers owned by the caller (except where stated);
 *     nothing is allocated, nothing is freed, the host never synchronises;
 *   - work is enqueued on `stream` (0 = legacy default stream) and is
 *     asynchronous; results are bitwise identical from run to run;
 *   - return 0 (MSA_OK) or an msa_status code; argument errors are detected
 *     on the host before anything is enqueued; MSA_ECUDA reports a launch error;
 *   - values that live on the device (seq_lens, selected block ids) cannot be
 *     checked on the host: kernels clamp or skip them and set a bit in the
 *     optional device status word (msa_params_t.status).
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MSA_BLOCK_TOKENS 128 /* tokens per MSA block */
#define MSA_TOPK_BLOCKS 16   /* blocks attended per query */

typedef enum msa_status {
    MSA_OK = 0,
    MSA_EINVAL = 1,       /* null pointer, non-positive size, bad tensor scale, lmax % 128 != 0 */
    MSA_EUNSUPPORTED = 2, /* shape outside what the kernels are built for (see msa_params_t) */
    MSA_EALIGN = 3,       /* a pointer is not 16-byte aligned */
    MSA_EWORKSPACE = 4,   /* workspace too small or NULL */
    MSA_ECUDA = 5         /* the CUDA runtime reported an error when launching */
} msa_status;

/* Bits of the optional device status word. */
#define MSA_STATUS_SEQLEN 1u   /* some seq_lens[b] < Tq or > lmax: clamped */
#define MSA_STATUS_SELECT 2u   /* a selected block id >= the visible block count: skipped */
#define MSA_STATUS_TIMEOUT 4u  /* a bounded wait inside a kernel gave up (results invalid) */
#define MSA_STATUS_PAGE 8u     /* a block-table page id outside the pool: page 0 read (results invalid) */
/* With MSA_STATUS_TIMEOUT, which wait gave up: */
#define MSA_STATUS_AT_INDEX_PRODUCER 0x100u /* indexer: producer waiting for a free stage */
#define MSA_STATUS_AT_INDEX_DRAIN 0x200u    /* indexer: producer draining its last copies */
#define MSA_STATUS_AT_INDEX_CONSUMER 0x400u /* indexer: consumer waiting for a stage's bytes */
#define MSA_STATUS_AT_ATTEND 0x800u         /* attention: warp waiting for its block's bytes */
#define MSA_STATUS_AT_DECODE_STAGE 0x1000u  /* single-launch decode: warp waiting for a stage's bytes */
#define MSA_STATUS_AT_DECODE_WAIT 0x2000u   /* single-launch decode: warp waiting for another warp's
                                               pooled scores or selection */

/* One NVFP4 cache tensor (K, V or index-K); the layout is given above.  With a
 * block table (msa_params_t.block_table) the planes are page pools instead:
 * data [num_pages][heads][128][dim/2], scale [num_pages][heads][128][dim/16]. */
typedef struct msa_nvfp4_cache {
    const uint8_t* data;  /* [B][heads][lmax][dim/2], 16-byte aligned */
    const uint8_t* scale; /* [B][heads][lmax][dim/16], 16-byte aligned */
    float tensor_scale;   /* > 0, finite */
} msa_nvfp4_cache_t;

/*
 * Problem description shared by every MSA entry point.
 *   B, Tq     sequences and query tokens per sequence (Tq >= 1)
 *   Hq, Hkv   attention query / KV heads; Hq / Hkv in {1, 2, 4, 8}
 *   D         attention head dim; 128
 *   HI, DI    indexer heads / dim; HI in {1, 2, 4, 8}, DI in {64, 128};
 *             Tq * HI <= 32 runs the decode indexer, larger Tq * HI (chunked
 *             prefill) the tensor-core indexer, which supports mean pooling
 *             only and no token_scores output
 *   lmax      cache capacity in tokens, a multiple of 128
 *   seq_lens  device int32 [B], Tq <= L_b <= lmax
 *   k, v      caches with Hkv heads of dim D; ik: 1 head of dim DI
 *   q         device bf16 [B][Tq][Hq][D]; q_idx: bf16 [B][Tq][HI][DI].  The
 *             kernels use queries as fp16: |q| must stay below 65504, and bf16
 *             values below 2^-14 in magnitude keep 11 significant bits at most
 *   w_idx     device fp32 [B][Tq][HI] indexer head weights, or NULL (all 1)
 *   softmax_scale  0 means 1/sqrt(D)
 *   pool_mode 0 = mean, 1 = max
 *   status    device uint32 status word (bits MSA_STATUS_*), or NULL; kernels
 *             only OR bits into it, the caller clears it
 *   block_table  NULL for contiguous caches; else a paged cache: device int32
 *             [B][lmax/128] mapping block n of sequence b to a page of the k, v
 *             and ik pools (one page = one 128-token MSA block of every head).
 *             A page id outside [0, num_pages) sets MSA_STATUS_PAGE and page 0
 *             is read in its place (results invalid)
 *   num_pages pages in each pool (> 0 with a block table)
 *   out_bf16  0: attention output fp32; 1: bf16 (the fp32 result rounded to
 *             nearest even, for the next layer); lse stays fp32
 */
typedef struct msa_params {
    int B, Tq, Hq, Hkv, D, HI, DI;
    int64_t lmax;
    const int32_t* seq_lens;
    msa_nvfp4_cache_t k, v, ik;
    const void* q;
    const void* q_idx;
    const float* w_idx;
    float softmax_scale;
    int pool_mode;
    uint32_t* status;
    const int32_t* block_table;
    int64_t num_pages;
    int out_bf16;
} msa_params_t;

/* Human-readable name of an msa_status code (static string, never NULL). */
const char* msa_status_string(int code);

/* Number of SMs etc. are queried once per device; this returns the library
 * build identification (static string). */
const char* msa_version(void);

/* ---------------------------------------------------------------------------
 * NVFP4 codec (the format of the readmex.ai TL;DR, "NVFP4 KV cache for both
 * the indexer and the attention path"; layout as above).
 * ------------------------------------------------------------------------- */

/* Quantise x (fp32 [nvec][dim], dim % 16 == 0) into NVFP4 planes:
 * per 16 elements s = E4M3_rne_sat(amax / fp32(6 * tensor_scale)),
 * code_i = E2M1_rne_sat(x_i / fp32(s * tensor_scale)) (all codes 0 when that
 * denominator is 0).  Inputs must be finite.  This is the cache write
 * ("KV-insert") that precedes the MSA path. */
int msa_nvfp4_encode(const float* x, int64_t nvec, int dim, float tensor_scale,
                     uint8_t* data, uint8_t* scale, cudaStream_t stream);

/* Dequantise NVFP4 planes into fp32 [nvec][dim]: fp32(e2m1 * e4m3) * tensor_scale. */
int msa_nvfp4_decode(const uint8_t* data, const uint8_t* scale, int64_t nvec, int dim,
                     float tensor_scale, float* out, cudaStream_t stream);

/* amax = max |x_i| over n fp32 values, written to *amax_out (device fp32).
 * A tensor scale for msa_nvfp4_encode is amax / (6 * 448). */
int msa_nvfp4_amax(const float* x, int64_t n, float* amax_out, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * MSA steps ("A model built for efficient inference", ainewsbites.com)
 * ------------------------------------------------------------------------- */

/* Bytes of scratch msa_decode needs for this problem (0 on invalid params): the pooled
 * block scores and the selection; for chunked prefill (Tq * HI > 32) with Hq = 8 * Hkv
 * also the per-block token lists and the per-(token, selected block) attention partials
 * of the tensor-core prefill attention, B * Tq * 16 * Hq * (2 D + 8) bytes and more
 * (about 1.15 GB for 2 sequences x 4,096 tokens x 32 heads on a 128K context). */
size_t msa_workspace_size(const msa_params_t* p);

/* Indexer + block pooling: streams every visible NVFP4 index key once.
 *   block_scores  fp32 [B][Tq][ceil(lmax/128)]: pooled score of each block,
 *                 -inf for blocks with no visible key
 *   token_scores  fp32 [B][Tq][lmax] or NULL: s_j for every visible key j
 *                 (entries of invisible keys are left untouched) */
int msa_index(const msa_params_t* p, float* block_scores, float* token_scores,
              cudaStream_t stream);

/* Top-16 block selection with the recent block forced:
 *   block_scores  fp32 [B][Tq][ceil(lmax/128)] as written by msa_index
 *   sel           int32 [B][Tq][16]: selected block ids ascending, -1 padded */
int msa_select(const msa_params_t* p, const float* block_scores, int32_t* sel,
               cudaStream_t stream);

/* Exact softmax attention over the selected blocks (split over the blocks,
 * combined in on-chip memory):
 *   sel  int32 [B][Tq][16] (ids < 0 are skipped)
 *   out  [B][Tq][Hq][D], fp32 (bf16 with out_bf16); lse fp32 [B][Tq][Hq] (natural log of the
 *        softmax denominator of the scaled scores) or NULL */
int msa_attend(const msa_params_t* p, const int32_t* sel, void* out, float* lse,
               cudaStream_t stream);

/* The whole MSA decode step: msa_index -> msa_select -> msa_attend (two
 * launches when the rows have <= 1,024 blocks: the selection then runs inside
 * the attention kernel).  For chunked prefill (Tq * HI > 32) with Hq = 8 * Hkv
 * the attention goes block by block on the tensor cores instead (the selection
 * inverted into per-block token lists, each block dequantised once per KV head,
 * tcgen05 tiles, the per-slot partials merged in slot order); results agree
 * with msa_attend's within the attention tolerance and are bitwise
 * reproducible.  Besides cudaMemsetAsync of a counter array in the workspace,
 * that path enqueues seven kernels.
 *   ws, ws_bytes  device scratch of at least msa_workspace_size(p) bytes,
 *                 256-byte aligned; contents on entry are ignored
 *   out, lse      as for msa_attend
 *   sel_out       int32 [B][Tq][16] copy of the selection, or NULL */
int msa_decode(const msa_params_t* p, void* ws, size_t ws_bytes, void* out, float* lse,
               int32_t* sel_out, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Indexer decode context parallelism (the pages' "DCP": "vLLM delivers day-0
 * support for MiniMax-M3.1-Flash", readmex.ai, TL;DR; "vLLM Adds Day-0 Support
 * for MiniMax-M3.1-Flash on NVIDIA and AMD GPUs", ainewsbites.com, "Kernel and
 * serving optimizations": the indexer of a long decode context is split over
 * GPUs).  The pages give no algorithm; this library's reading keeps the
 * single-GPU result:
 *
 *   G ranks split the blocks of every sequence into G contiguous ranges that
 *   cover [0, lmax/128) without overlap; rank g holds blocks [n0, n1) of the K,
 *   V and index-K caches (contiguous caches of full capacity of which only the
 *   range is read, or a paged cache whose block table names pages only for the
 *   range: entries outside it are never read).  One decode step is
 *     msa_dcp_candidates (own range) -> all-gather of the candidates ->
 *     msa_dcp_merge (same result on every rank) -> msa_dcp_attend (own range)
 *     -> all-gather of the partials -> msa_dcp_combine.
 *   The merged selection equals msa_decode's bit for bit (every block's pooled
 *   score is computed by the same arithmetic; the best 15 blocks of the context
 *   are among the ranks' best 15); the combined output matches msa_decode's
 *   within the attention tolerance (the partials are merged in another order).
 *   Exchanged bytes per query row: G x 16 x 8 (candidates) and
 *   G x Hq x (D + 1) x 4 (partials).  The exchange itself is the caller's (NCCL
 *   all-gather in the package's Python layer); these calls only compute.
 *   Decode indexer only: Tq * HI <= 32.  Results are bitwise deterministic.
 * ------------------------------------------------------------------------- */

/* Scratch for msa_dcp_candidates: the pooled block scores [B][Tq][lmax/128] fp32. */
size_t msa_dcp_workspace_size(const msa_params_t* p);

/* The indexer and block pooling over blocks [n0, n1) only (0 <= n0 < n1 <= lmax/128),
 * then, per (sequence, query token), this rank's candidates: its best min(15, c)
 * blocks other than the query's own block r (c = the visible blocks of the range
 * other than r), by (score desc, block index asc):
 *   ws, ws_bytes  at least msa_dcp_workspace_size(p) bytes, 256-byte aligned
 *   cand_score    fp32 [B][Tq][16], cand_id int32 [B][Tq][16]: the candidates
 *                 (ascending block order for ranges of up to 4,096 blocks, else by
 *                 descending score; the merge does not depend on the order), then
 *                 (-inf, -1) padding (slot 15 is always padding)
 * Returns MSA_EINVAL for an empty or out-of-bounds range, MSA_EUNSUPPORTED for
 * Tq * HI > 32. */
int msa_dcp_candidates(const msa_params_t* p, int64_t n0, int64_t n1, void* ws, size_t ws_bytes,
                       float* cand_score, int32_t* cand_id, cudaStream_t stream);

/* Merge of G ranks' candidates (1 <= G <= 32), every rank the same way:
 *   cand_score fp32 [G][B][Tq][16], cand_id int32 [G][B][Tq][16] (rank g's
 *   msa_dcp_candidates output at index g)
 *   sel        int32 [B][Tq][16]: the query's own block plus the best min(15, r)
 *              pairs by (score desc, id asc), ascending, -1 padded.  Pairs whose id
 *              is not a visible block other than r are ignored; a pair received
 *              twice counts once. */
int msa_dcp_merge(const msa_params_t* p, int G, const float* cand_score, const int32_t* cand_id,
                  int32_t* sel, cudaStream_t stream);

/* Attention of every query over those of its selected blocks that lie in [n0, n1):
 *   out  fp32 [B][Tq][Hq][D], normalised over this rank's keys (zeros when the
 *        rank holds none of the query's selected blocks); out_bf16 is ignored
 *   lse  fp32 [B][Tq][Hq] (required): natural log of the softmax denominator over
 *        this rank's keys, -inf when it holds none of them */
int msa_dcp_attend(const msa_params_t* p, int64_t n0, int64_t n1, const int32_t* sel, float* out, float* lse,
                   cudaStream_t stream);

/* Combine of G partials (1 <= G <= 32) in rank order:
 *   part_out fp32 [G][B][Tq][Hq][D], part_lse fp32 [G][B][Tq][Hq]
 *   out      [B][Tq][Hq][D], fp32 (bf16 with out_bf16): sum_g exp(lse_g - lse) out_g
 *   lse      fp32 [B][Tq][Hq] or NULL: log sum_g exp(lse_g) */
int msa_dcp_combine(const msa_params_t* p, int G, const float* part_out, const float* part_lse, void* out,
                    float* lse, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * The decode step as one persistent launch.  Prior art: the single-launch
 * "mono" decode path of "vLLM turns MiniMax's day-zero promise into
 * GPU-specific serving code" (upstreambeat.ai, "What changed").  Same results
 * as msa_decode (same selection; attention within the stated tolerance, the
 * per-block partials being combined in another order).  Every warp of the grid
 * works through one list of index, select and attention items, so the
 * attention of early sequences overlaps the index stream of later ones.  On
 * B200 at the decode workloads of this library it is slower than msa_decode
 * (each select and attention item is a chain on one warp, where the separate
 * kernels spread the same work over 16 warps); it is kept as a measured
 * alternative, not used by msa_decode.
 * ------------------------------------------------------------------------- */

/* Scratch for msa_decode_single_launch (0 if the problem is not supported:
 * it needs Tq * HI <= 16 and contiguous caches): counters, pooled scores,
 * selection and per-block attention partials. */
size_t msa_workspace_size_single_launch(const msa_params_t* p);

/* As msa_decode, in one launch (plus one cudaMemsetAsync that clears the
 * workspace's counter region on `stream`).
 *   ws, ws_bytes  at least msa_workspace_size_single_launch(p) bytes,
 *                 256-byte aligned; contents on entry are ignored; one call
 *                 at a time may use it
 * Returns MSA_EUNSUPPORTED for Tq * HI > 16 or a block table.  A wait inside the kernel for
 * another warp's result that exceeds 2 s (all CTAs of the grid must be
 * resident: another kernel holding SMs for that long) sets MSA_STATUS_TIMEOUT
 * | MSA_STATUS_AT_DECODE_WAIT and ends the launch. */
int msa_decode_single_launch(const msa_params_t* p, void* ws, size_t ws_bytes, void* out,
                             float* lse, int32_t* sel_out, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Decode without caller scratch.  No counterpart in the paper: this is a
 * convenience of this library for callers that cannot allocate device memory.
 * ------------------------------------------------------------------------- */

/* Size of the library-owned device scratch array used by msa_decode_static. */
#define MSA_STATIC_SCRATCH_BYTES (4u << 20) /* 4 MiB */

/* msa_decode with its scratch (block scores + selection) in a fixed device
 * array of MSA_STATIC_SCRATCH_BYTES owned by the library, for callers that
 * cannot call cudaMalloc: a plugin handed only its inputs and outputs by a host
 * framework that owns all device memory, or a hot loop that must not risk the
 * device-wide synchronisation an allocation can cause.  Calls no allocation
 * routine, on the device or the host (but see the first-call note below).
 *   p, out, lse, sel_out, stream   as for msa_decode
 * Returns the msa_decode argument errors, or MSA_EWORKSPACE when
 * msa_workspace_size(p) exceeds MSA_STATIC_SCRATCH_BYTES (e.g. B * Tq *
 * lmax / 128 * 4 bytes of block scores beyond about 4 MiB), or MSA_ECUDA if
 * the array's device address cannot be obtained.
 * Notes:
 *   - every GPU that loads libmsa.so holds the array until the process exits;
 *   - the first call on each device looks up the array's address (once, with
 *     that device current).  With lazy module loading (the CUDA default) the
 *     driver only loads the library's module, and so places the array in
 *     device memory, at that lookup: the first call may therefore allocate on
 *     the driver's side and synchronise.  Treat it as the warm-up call, and
 *     make it before any stream capture and outside latency-critical code;
 *   - after cudaDeviceReset the next call looks the address up again (the
 *     device then has a new context and the array a new address);
 *   - all calls share the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other host threads) race
 *     and must be serialised by the caller. */
int msa_decode_static(const msa_params_t* p, void* out, float* lse, int32_t* sel_out,
                      cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* MSA_H */
