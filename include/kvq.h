/*
 * kvq.h -- C ABI of libkvq.so: a sub-4-bit KVQuant KV cache on NVIDIA B200 (sm_100a).
 *
 * The library implements the decode-time hot path of KVQuant ("KVQuant: Towards
 * 10 Million Context Length LLM Inference with KV Cache Quantization", arXiv
 * 2401.18079):
 *   - the append-time quantizer that writes the cache, using (i) per-channel key
 *     quantization, (ii) pre-RoPE keys, (iii) a per-layer non-uniform (NUQ)
 *     datatype and (iv) per-vector dense-and-sparse outliers (study.space
 *     summary, techniques (i)-(iv); phantomic12 research note, components (1)-(4));
 *   - decode attention read directly from that cache: QK with on-the-fly NUQ
 *     lookup, RoPE and sparse outlier correction, a split-K softmax with a
 *     max/sum merge, and the probability-weighted value sum (study.space
 *     summary: custom kernels replacing the fp16 matrix-vector products of
 *     memory- and bandwidth-bound long-context decode).
 *
 * Conventions (every entry point):
 *   - Buffers are DEVICE pointers owned by the caller unless a parameter says
 *     "host".  Cache and workspace buffers must be 16-byte aligned.  The library
 *     allocates no device buffer; its only global state is the fixed scratch array of
 *     kvq_quantize_append_noalloc and the per-thread text of the last CUDA error
 *     (a kvq_step owns host memory and an instantiated CUDA graph).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls only enqueue work; none synchronizes except kvq_get_status.
 *   - Return value: KVQ_OK (0) or a negative KVQ_ERR_* code.  Argument checks are
 *     synchronous and nothing is launched when one fails.  KVQ_ERR_CUDA reports
 *     a failed launch; the CUDA error string is available via kvq_strerror.
 *   - Conditions only the device can see (an outlier list that is full, a length
 *     past T_max) set bits in the sticky int32 `status` word of the cache and the
 *     kernel carries on without trapping; read it with kvq_get_status.
 *   - fp16 values travel as their uint16_t bit patterns.
 *   - Only head_dim D = 128 and bits in {2, 3, 4} are supported.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_ABI_VERSION 2

enum {
    KVQ_OK = 0,
    KVQ_ERR_NULL = -1,        /* a required pointer is NULL */
    KVQ_ERR_ALIGN = -2,       /* a device pointer is not 16-byte aligned */
    KVQ_ERR_SHAPE = -3,       /* a dimension or count is out of range */
    KVQ_ERR_UNSUPPORTED = -4, /* bits or head_dim not supported */
    KVQ_ERR_RANGE = -5,       /* token range beyond T_max / split count out of range */
    KVQ_ERR_WORKSPACE = -6,   /* workspace smaller than the size query returned */
    KVQ_ERR_CUDA = -7,        /* a CUDA launch or runtime call failed */
    KVQ_ERR_SCRATCH_LIMIT = -8, /* request exceeds the fixed scratch of kvq_quantize_append_noalloc */
};

/* Sticky device status bits (cache->status). */
#define KVQ_STATUS_OUTLIER_OVERFLOW 1 /* outliers of some tokens did not fit and were dropped */
#define KVQ_STATUS_LEN_OVERFLOW 2     /* a write past T_max (or a length past max_len) was skipped */
#define KVQ_STATUS_NOT_EMPTY 4        /* a calibrating prefill met a non-empty sequence; skipped */
#define KVQ_STATUS_WAIT_TIMEOUT 8     /* a decode kernel gave up waiting for its bulk copies; its
                                         outputs of that call are invalid */
#define KVQ_STATUS_SMEM_LAYOUT 16     /* the fused decode kernel found its shared-memory window
                                         based too high for its table layout; its outputs of that
                                         call are invalid */
#define KVQ_STATUS_CODEBOOK 32        /* the fused decode kernel met value levels that are not of
                                         the (u << 16) | u form; its outputs are invalid */

#define KVQ_CHUNK 64 /* tokens per outlier chunk */

/* Geometry of one layer's cache.  n = Hkv * D channels per token. */
typedef struct kvq_cfg {
    int32_t B;          /* sequences (batch) */
    int32_t Hq;         /* query heads; a multiple of Hkv */
    int32_t Hkv;        /* key/value heads */
    int32_t D;          /* head dimension; must be 128 */
    int32_t bits;       /* NUQ code width: 2, 3 or 4 */
    int32_t T_max;      /* token capacity per sequence, 1 .. 16,777,216 */
    int32_t out_cap_k;  /* key-outlier list capacity per (sequence, kv head); multiple of 8 */
    int32_t out_cap_v;  /* value-outlier list capacity per (sequence, kv head); multiple of 8 */
    double outlier_frac;/* f: per vector, k = floor(f*N/2 + 1/2) outliers per side */
    double rope_theta;  /* RoPE base; theta_i = rope_theta^(-2i/D) */
} kvq_cfg;

/*
 * Device arrays of one layer's cache (all caller-allocated; sizes from kvq_layout).
 * Layouts (codes are little-endian bit strings over consecutive uint32 words):
 *  kcodes, vcodes  uint32 [B][Hkv][ceil(T_max/4)][16*bits]  one code block per (sequence,
 *          kv head, token quad 4u .. 4u+3), keys and values alike.  Lane group i in [0,16)
 *          owns words [bits*i, bits*i + bits) of the block and the rotate-half pairs
 *          (c, c + 64), c = i + 16k (k in [0,4)).  Token j of the quad sits in slot
 *          s = j ^ (i >> 2): the 2*bits-wide field at bit 2*bits*(4k + s) of the group's
 *          bit string holds code(4u + j, c) | code(4u + j, c + 64) << bits.  Fields of
 *          tokens not yet written are 0.
 *  kthr    uint16 [B][n][2]  fp16 key thresholds (t_lo, t_hi) per channel
 *  kparams float  [B][n][2]  key channel (off, half)
 *  vparams float  [B][T_max][2] value token (off, half)
 *  kout, vout uint32 [B][Hkv][cap]  one outlier list per (sequence, kv head): entry
 *          (fp16 bits << 16) | ((t % 64) << 7) | c (c the channel within the head),
 *          sorted by (t, c)
 *  k/vchunk uint32 [B][Hkv][ceil(T_max/64)+1]  entries of tokens [64m, 64m+64) are
 *          [chunk[m], chunk[m+1])
 *  k/vcount uint32 [B][Hkv]  entries in use;  len int32 [B]  tokens in the cache
 *  status  int32 [1]  sticky KVQ_STATUS_* bits
 */
typedef struct kvq_cache {
    uint32_t* kcodes;
    uint32_t* vcodes;
    uint16_t* kthr;
    float* kparams;
    float* vparams;
    uint32_t* kout;
    uint32_t* vout;
    uint32_t* kchunk;
    uint32_t* vchunk;
    uint32_t* kcount;
    uint32_t* vcount;
    int32_t* len;
    int32_t* status;
} kvq_cache;

/* A per-layer NUQ datatype (device arrays): levels[2^bits] ascending binary32
 * values whose bit patterns are (u << 16) | u, and the decision bounds
 * bounds[2^bits - 1] = binary32((levels[j] + levels[j+1]) / 2). */
typedef struct kvq_codebook {
    const float* levels;
    const float* bounds;
} kvq_codebook;

/* Byte size of every cache array of kvq_cache, same field names. */
typedef struct kvq_sizes {
    size_t kcodes, vcodes, kthr, kparams, vparams;
    size_t kout, vout;
    size_t kchunk, vchunk, kcount, vcount, len, status;
} kvq_sizes;

/* ABI version (KVQ_ABI_VERSION). */
int kvq_abi_version(void);

/* Static message for a KVQ_* code; for KVQ_ERR_CUDA the last CUDA error's text.
 * The pointer is owned by the library and valid until the next call. */
const char* kvq_strerror(int code);

/* Check a configuration.  KVQ_OK, KVQ_ERR_NULL, KVQ_ERR_SHAPE or KVQ_ERR_UNSUPPORTED. */
int kvq_validate_cfg(const kvq_cfg* cfg);

/* Fill *out (host) with the byte size of each cache array for cfg. */
int kvq_layout(const kvq_cfg* cfg, kvq_sizes* out);

/* Empty the cache: zero len, counts, chunk pointers and status (async on stream). */
int kvq_cache_reset(const kvq_cfg* cfg, const kvq_cache* cache, void* stream);

/* Workspace bytes for kvq_quantize_append with this many tokens per sequence. */
int kvq_quantize_workspace(const kvq_cfg* cfg, int32_t n_new, int32_t calibrate, size_t* bytes);

/*
 * Quantize and append tokens (technique (i)-(iv) on the write side).
 *   k, v     fp16 [B][n_new][Hkv][D] pre-RoPE keys and values (device, 16-byte
 *            aligned; KVQ_ERR_ALIGN otherwise)
 *   plen     int32 [B] tokens of sequence b to take from the block (<= n_new),
 *            or NULL for n_new each (device)
 *   calibrate 1: prefill -- the sequence must be empty; per key channel the
 *            thresholds t_lo = s[k], t_hi = s[N-1-k] of its N = plen[b] values
 *            (ascending in IEEE total order, k = floor(f*N/2 + 1/2) capped at
 *            (N-1)/2) and off = (t_lo+t_hi)*0.5, half = (t_hi-t_lo)*0.5 (binary32)
 *            are computed first.  0: append at positions len[b] onwards with the
 *            existing key calibration.
 *   Per token: value thresholds/scales over its n values as above; an entry is
 *   an outlier iff x < t_lo or x > t_hi; outliers go to the lists unchanged and
 *   are encoded as 0; xn = (x - off)/half (0 if half == 0); code = #{j: xn >
 *   bounds[j]}.  Per list (sequence, kv head): a token whose outliers in that head
 *   would exceed the list capacity (counting from the start of this call, in token
 *   order) drops them there and sets KVQ_STATUS_OUTLIER_OVERFLOW.
 *   workspace: device scratch of kvq_quantize_workspace bytes, 16-byte aligned.
 */
int kvq_quantize_append(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                        const kvq_codebook* cbV, const uint16_t* k, const uint16_t* v,
                        int32_t n_new, const int32_t* plen, int32_t calibrate, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * Decode QK (technique (ii) read side): for every query head hq (kv head
 * h = hq / (Hq/Hkv)) and cached token t < len[b]:
 *   logits[b][hq][t] = (R(qpos[b]) q) . (R(t) khat_t,h) / sqrt(D)
 * with rotate-half RoPE R and khat the dequantized key (dense off + half*L[code],
 * outliers replaced by their stored value).  Also writes per split s (tokens
 * [s*Ls, (s+1)*Ls), Ls = the split length chosen from max_len and `splits`):
 *   stats[b][hq][s] = (m_s, l_s), m_s = max logit, l_s = sum exp(logit - m_s)
 * (m_s = -inf, l_s = 0 for an empty split).
 *   q       fp16 [B][Hq][D] pre-RoPE query;  qpos int32 [B] its position
 *   max_len host upper bound on len[b] (sizes the grid); a longer sequence is
 *           clipped and sets KVQ_STATUS_LEN_OVERFLOW
 *   logits  float [B][Hq][T_max];  stats float2 [B][Hq][splits]
 *   splits  1 .. 4096, or 0 to let the library choose (kvq_decode_splits)
 *   workspace  device scratch of kvq_decode_qk_workspace bytes (per-call tables: the
 *           rotated query, RoPE angle tables, the dense key value at outliers), 16-byte
 *           aligned
 */
int kvq_decode_qk(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                  const uint16_t* q, const int32_t* qpos, int32_t max_len, float* logits,
                  float* stats, int32_t splits, void* workspace, size_t workspace_bytes,
                  void* stream);

/* Workspace bytes of kvq_decode_qk for max_len. */
int kvq_decode_qk_workspace(const kvq_cfg* cfg, int32_t max_len, size_t* bytes);

/* The split count the library uses for `splits = 0`. */
int kvq_decode_splits(const kvq_cfg* cfg, int32_t max_len);

/*
 * Split-K softmax merge (the softmax of decode attention, done by the custom decode
 * kernels that read the quantized cache directly: study.space summary, custom CUDA
 * kernels for memory- and bandwidth-bound long-context decode).  The pages fix the
 * softmax, not how it is split; the split into token ranges is this library's, and the
 * merge is the exact identity softmax(l) over the union of the ranges:
 *   ml[b][hq] = (M, L), M = max_s m_s, L = sum_s l_s e^(m_s - M)   (binary32).
 *   stats float2 [B][Hq][splits] from kvq_decode_qk (device); ml float2 [B][Hq] (device)
 * An empty split (m_s = -inf, l_s = 0) contributes nothing; all splits empty gives
 * (-inf, 0).  Errors: KVQ_ERR_NULL, KVQ_ERR_RANGE (splits outside 1 .. 4096).
 */
int kvq_softmax_merge(const kvq_cfg* cfg, const float* stats, int32_t splits, float* ml,
                      void* stream);

/*
 * Decode PV (the value half of the custom decode kernels, study.space summary; the
 * read side of per-token value quantization onto the NUQ datatype, technique (iii),
 * with per-vector dense-and-sparse outliers, technique (iv); phantomic12 research
 * note, components (3) and (4)):
 *   out[b][hq][:] = sum_t p_t * vhat_t,h with p_t = exp(logits - M)/L and
 * vhat the dequantized value (off_t + half_t*L[code], outliers replaced).  The sum over
 * the outlier entries of each output is taken in a fixed order, so two calls on the same
 * inputs return the same bits.
 *   logits, ml from the two calls above; out float [B][Hq][D]
 *   part   float scratch [B][Hq][splits][D] (per-split partial sums, summed in
 *          split order)
 * A sequence with no cached token (len 0) gets out = 0.
 */
int kvq_decode_pv(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbV,
                  const float* logits, const float* ml, int32_t max_len, float* out, float* part,
                  int32_t splits, void* stream);

/* Workspace bytes of kvq_decode_attention for max_len and splits (0 = auto). */
int kvq_decode_workspace(const kvq_cfg* cfg, int32_t max_len, int32_t splits, size_t* bytes);

/*
 * Decode attention in one call: kvq_decode_qk, kvq_softmax_merge and kvq_decode_pv
 * on `stream`, with their buffers (logits [B][Hq][T_max], split statistics, (M, L),
 * split partials, per-call tables) carved from `workspace`; the same result as the
 * three calls, the same bits on every run; out float [B][Hq][D].
 *   workspace  device scratch of kvq_decode_workspace bytes, 16-byte aligned
 */
int kvq_decode_attention(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                         const kvq_codebook* cbV, const uint16_t* q, const int32_t* qpos,
                         int32_t max_len, float* out, void* workspace, size_t workspace_bytes,
                         int32_t splits, void* stream);

/*
 * Decode attention over one token range of a longer sequence, as a partial for a merge: the
 * building block of the token-sharded decode (the pages' "10 million context across 8 GPUs":
 * study.space summary; phantomic12 research note, the consequence claim).  A device holds
 * tokens [pos_offset, pos_offset + len[b]) of sequence b in `cache` (row t of the cache sits at
 * position pos_offset + t; RoPE uses that position) and computes, per (b, hq),
 *   ml[b][hq] = (M, L), M = max_t l_t, L = sum_t e^(l_t - M),
 *   o[b][hq][:] = sum_t e^(l_t - M) vhat_t       (not divided by L),
 * with l_t, vhat_t exactly as kvq_decode_attention; an empty range gives (-inf, 0) and o = 0.
 *   pos_offset  host int32 >= 0 (the same for every sequence of the batch)
 *   ml float2 [B][Hq], o float [B][Hq][D] (device); workspace as kvq_decode_workspace
 * kvq_decode_partial followed by kvq_merge_partials over all ranges equals
 * kvq_decode_attention over the whole sequence up to rounding.
 */
int kvq_decode_partial(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                       const kvq_codebook* cbV, const uint16_t* q, const int32_t* qpos,
                       int32_t max_len, int32_t pos_offset, float* ml, float* o,
                       void* workspace, size_t workspace_bytes, int32_t splits, void* stream);

/*
 * Merge of `parts` partials of kvq_decode_partial (the softmax over the union of their token
 * ranges, an exact identity): out[b][hq][:] = sum_k e^(M_k - M) o_k / sum_k e^(M_k - M) L_k,
 * M = max_k M_k, taken in part order; 0 when no part has a token.
 *   ml float2 [parts][B][Hq], o float [parts][B][Hq][D], out float [B][Hq][D] (device)
 * Errors: KVQ_ERR_NULL, KVQ_ERR_RANGE (parts outside 1 .. 4096).
 */
int kvq_merge_partials(const kvq_cfg* cfg, int32_t parts, const float* ml, const float* o,
                       float* out, void* stream);

/*
 * Decode attention in one fused pass per (split, sequence, head): QK with NUQ lookup and RoPE,
 * the key-outlier correction, an online softmax, PV and the value-outlier correction in one
 * kernel, then the split merge (the custom decode kernels of the study.space summary, here
 * without a logits buffer).  The same result as kvq_decode_attention up to rounding, summed in
 * a fixed order (the same bits on every run).  For kv heads that serve one query head each
 * (Hq == Hkv) and bits 2 or 3 (KVQ_ERR_UNSUPPORTED otherwise); the value levels must have the
 * (u << 16) | u form the codebook contract states (else KVQ_STATUS_CODEBOOK is set).
 *   workspace  kvq_decode_fused_workspace bytes: no [B][Hq][T_max] logits, so far smaller
 *              than kvq_decode_workspace at long contexts (134 MB less at 2^20 tokens x 32 heads)
 */
int kvq_decode_attention_fused(const kvq_cfg* cfg, const kvq_cache* cache,
                               const kvq_codebook* cbK, const kvq_codebook* cbV,
                               const uint16_t* q, const int32_t* qpos, int32_t max_len,
                               float* out, void* workspace, size_t workspace_bytes,
                               int32_t splits, void* stream);

/* Workspace bytes of kvq_decode_attention_fused (KVQ_ERR_UNSUPPORTED for other shapes). */
int kvq_decode_fused_workspace(const kvq_cfg* cfg, int32_t max_len, int32_t splits,
                               size_t* bytes);

/*
 * Dequantize rows [t0, t0 + nt) of every sequence (test support):
 *   khat, vhat fp16 [B][nt][Hkv][D] (keys pre-RoPE): dense fp16(off + half*L[code])
 *   (binary32 multiply, then add, then round to fp16), outliers replaced by their
 *   stored fp16 value.  Rows at or past len[b] are written as 0.
 */
int kvq_dequantize(const kvq_cfg* cfg, const kvq_cache* cache, const kvq_codebook* cbK,
                   const kvq_codebook* cbV, int32_t t0, int32_t nt, uint16_t* khat,
                   uint16_t* vhat, void* stream);

/*
 * Uncompressed comparison kernel: decode attention over an fp16 cache.  The pages
 * measure the KVQuant kernels against fp16 matrix-vector multiplication (study.space
 * summary, "~1.7x" over the fp16 baseline); this is that baseline, written for the
 * same layouts and the same RoPE reading, so the two can be timed side by side.
 *   K, V fp16 [B][T_stride][Hkv][D] (keys pre-RoPE, RoPE applied on the fly);
 *   len int32 [B]; q, qpos as kvq_decode_qk; out float [B][Hq][D];
 *   workspace of kvq_decode_workspace bytes for the same cfg/max_len/splits.
 * Hq/Hkv must be 1, 2, 4 or 8 (KVQ_ERR_UNSUPPORTED otherwise).
 */
int kvq_fp16_decode_attention(const kvq_cfg* cfg, const uint16_t* K, const uint16_t* V,
                              int32_t T_stride, const int32_t* len, const uint16_t* q,
                              const int32_t* qpos, int32_t max_len, float* out, void* workspace,
                              size_t workspace_bytes, int32_t splits, void* stream);

/* Workspace bytes of kvq_fit_codebook. */
int kvq_fit_workspace(int32_t n_vec, int32_t vec_len, size_t* bytes);

/*
 * Fit a per-layer NUQ datatype (technique (iii)) on the device.
 *   samples fp16 [n_vec][vec_len]: each vector is thresholded and normalized by
 *   its own order statistics (as in kvq_quantize_append), its outliers are
 *   dropped, and the pooled normalized values (binary64) are fitted by weighted
 *   1-D Lloyd k-means with 2^bits centroids: init at weighted quantiles
 *   (j+1/2)/K, nearest centroid with ties to the lower index, weighted-mean
 *   update (an empty cell keeps its value), stop when the assignment repeats or
 *   after max_iter iterations.  Centroids are sorted, rounded to the nearest
 *   (u << 16) | u binary32 value and bounds are binary32 midpoints.
 *   weights  binary64 [n_vec][vec_len] sensitivity weights, or NULL for 1
 *   levels   float [2^bits], bounds float [2^bits - 1] (device outputs)
 *   n_vec * vec_len <= 16384.  Runs as one thread block.
 */
int kvq_fit_codebook(const uint16_t* samples, int32_t n_vec, int32_t vec_len, double f,
                     const double* weights, int32_t bits, int32_t max_iter, float* levels,
                     float* bounds, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Append tokens without any device allocation and without a workspace argument.
 * (No counterpart in the KVQuant pages: this is a deployment convenience of this library.)
 *
 * For callers that must not allocate device memory on their decode path: serving loops
 * that keep the allocator out of the per-token step for latency, runtimes that reserve a
 * fixed device-memory budget up front and hand plug-ins only pre-sized buffers, or code
 * that has no access to an allocator at all.  It does exactly what
 * kvq_quantize_append(..., calibrate = 0, ...) does, with its scratch taken from a
 * file-scope device array of KVQ_NOALLOC_SCRATCH_BYTES that the library owns; every GPU
 * that loads libkvq.so holds that array until the process exits.
 *   - Limit: the scratch that kvq_quantize_workspace(cfg, n_new, 0) reports must fit in
 *     KVQ_NOALLOC_SCRATCH_BYTES (1 MiB).  A call needs about 80 bytes per (sequence, new
 *     token) and 16*(n_new/64 + 2) + 32 bytes per (sequence, kv head): 256 sequences with
 *     32 kv heads fit appending up to 25 tokens each; larger requests return
 *     KVQ_ERR_SCRATCH_LIMIT and launch nothing.  Use kvq_quantize_append with a caller
 *     workspace for prefills.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before any
 *     stream capture begins.
 *   - All calls share the one array: calls that may run concurrently on the same GPU
 *     (different streams without ordering) race on it and must not be issued that way.
 *     Each call writes every scratch entry before reading it, so nothing needs clearing
 *     between calls.
 * Arguments, layouts and device-side status behaviour are those of kvq_quantize_append.
 */
#define KVQ_NOALLOC_SCRATCH_BYTES (1u << 20)
int kvq_quantize_append_noalloc(const kvq_cfg* cfg, const kvq_cache* cache,
                                const kvq_codebook* cbK, const kvq_codebook* cbV,
                                const uint16_t* k, const uint16_t* v, int32_t n_new,
                                const int32_t* plen, void* stream);

/*
 * Whole-model decode step as one CUDA graph.  The pages use the cache for token-by-token
 * generation over a long context on one GPU (study.space summary: LLaMA-7B served with a
 * context of a million tokens on a single GPU; phantomic12 research note, the paper's own
 * claim): for every generated token, every layer appends that token's key and value to its
 * cache and attends over the whole cache.  kvq_step_create records that step for `layers`
 * caches in one CUDA graph -- for l = 0 .. layers-1 in order, kvq_quantize_append
 * (calibrate = 0) of n_new tokens per sequence into caches[l] (nothing when n_new = 0), then
 * kvq_decode_attention (kvq_decode_attention_fused when desc->fused = 1) over caches[l] into
 * out[l] -- and kvq_step_launch replays it: one graph launch in place of about ten kernel
 * launches per layer.  A launch gives the same bits as those calls made one by one on the
 * same inputs.  (The layers' query, key and value inputs arrive together; the projections
 * that would produce them from the previous layer are model code, outside this library.)
 *
 * Inputs of a launch: one packed record of kvq_step_input_bytes bytes, which
 * kvq_step_launch copies into desc->inputs (the graph reads its inputs only there):
 *   for l = 0 .. layers-1:  k fp16 [B][n_new][Hkv][D], v fp16 [B][n_new][Hkv][D],
 *                           q fp16 [B][Hq][D]   (each part a multiple of 256 bytes)
 *   then qpos int32 [B] (each sequence's query position), padded to 16 bytes.
 * Each launch advances len[b] of every cache by n_new on the device.  desc->max_len sizes
 * the grids once, at create: it must bound len[b] after the append at every launch (a
 * longer sequence is clipped and sets KVQ_STATUS_LEN_OVERFLOW, as in kvq_decode_qk), and a
 * max_len far above the actual lengths costs empty splits.  Launches of one step share
 * desc->inputs, desc->out and the workspace: issue them on one stream, in order.
 */
typedef struct kvq_step kvq_step; /* opaque: the instantiated graph and its buffers */

typedef struct kvq_step_desc {
    int32_t layers;              /* 1 .. 4096 */
    const kvq_cache* caches;     /* host array [layers]; read during kvq_step_create only */
    const kvq_codebook* cbK;     /* host array [layers] (key datatypes) */
    const kvq_codebook* cbV;     /* host array [layers] (value datatypes) */
    int32_t n_new;               /* tokens appended per sequence and launch, 0 .. T_max */
    int32_t max_len;             /* 1 .. T_max, see above */
    int32_t splits;              /* as for kvq_decode_attention (0 = the library's choice) */
    int32_t fused;               /* 0 or 1 (kvq_decode_attention_fused) */
    void* inputs;                /* device, kvq_step_input_bytes bytes, 16-byte aligned */
    float* out;                  /* device float [layers][B][Hq][D], 16-byte aligned */
    void* workspace;             /* device scratch of kvq_step_workspace bytes, 16-byte aligned */
    size_t workspace_bytes;
} kvq_step_desc;

/* Bytes of one packed input record. */
int kvq_step_input_bytes(const kvq_cfg* cfg, int32_t layers, int32_t n_new, size_t* bytes);

/* Workspace bytes of a step: the append's scratch, then the attention's (layers share both,
 * since the recorded calls run one after another). */
int kvq_step_workspace(const kvq_cfg* cfg, int32_t n_new, int32_t max_len, int32_t splits,
                       int32_t fused, size_t* bytes);

/*
 * Record and instantiate the step.  Every recorded call checks its arguments here; on an
 * error the code is returned, *step is NULL and nothing has run on the GPU (recording runs
 * nothing).  The step owns host memory and the instantiated graph until kvq_step_destroy;
 * the library allocates no device buffer for it.  The graph is recorded (by stream capture in
 * relaxed mode, on a stream the call creates and destroys) for the calling thread's current
 * CUDA device, which must hold every buffer the descriptor names; launch it on a stream of
 * that device.
 */
int kvq_step_create(const kvq_cfg* cfg, const kvq_step_desc* desc, kvq_step** step);

/*
 * One step: copy the packed record `inputs` (host or device memory; NULL if the caller has
 * already written desc->inputs) into desc->inputs with cudaMemcpyAsync on `stream`, then
 * launch the graph on `stream`.  Enqueue only (a pageable host record is copied before the
 * call returns; a pinned one asynchronously, so keep it unchanged until the step completes).
 */
int kvq_step_launch(kvq_step* step, const void* inputs, void* stream);

/* Release the step.  Call it after the step's launches have completed. */
int kvq_step_destroy(kvq_step* step);

/* Read the sticky status word into *out (host).  Synchronizes `stream`. */
int kvq_get_status(const kvq_cache* cache, int32_t* out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* KVQ_H */
