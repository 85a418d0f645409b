/*
 * kvq.h -- C ABI of a few-bit KV-cache codec with decode attention on the packed cache,
 * written for NVIDIA B200 (sm_100a).
 *
 * What the library computes (cited by page title and section):
 *
 *  - "TurboQuant vs OSCAR vs EpiCache" (dothoosh.com), section "Quantization frontiers:
 *    TurboQuant and OSCAR". Stage one rotates each key/value vector at random so that its
 *    coordinates become close to independent Gaussians, then codes every coordinate with a
 *    precomputed Lloyd-Max scalar quantizer. Stage two sketches the residual with a 1-bit
 *    quantized Johnson-Lindenstrauss transform (QJL), which gives an unbiased estimate of the
 *    attention logit. The same section describes KIVI (keys per channel, values per token).
 *    The random rotation here is a randomized Hadamard transform R = H D / sqrt(d): D is a
 *    +-1 diagonal and H the Sylvester-Hadamard matrix (natural order).
 *  - Same page, section "KV-cache bottleneck": each decode step streams the whole cache, so
 *    decode attention is bound by HBM bandwidth.
 *  - "TaSQ 1-bit KV cache compression boosts batch sizes 14x": a cache of one sign bit per
 *    coordinate (here: rotation, one sign bit per coordinate, an fp16 norm).
 *  - "How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2", sections "CSA2" (one
 *    512-dim latent per token shared by every head) and "Numerics and hardware efficiency"
 *    (FP4 E2M1 storage with one scale per 16 channels; here the scale is an E4M3 byte).
 *
 * Conventions for every call:
 *  - Calls return a kvq_status and never abort or throw. Arguments are validated before any
 *    launch; a call that fails validation writes nothing.
 *  - A cache belongs to the CUDA device that was current when kvq_cache_init ran; calls that
 *    launch work on it return KVQ_ERR_INVALID_ARG, launching nothing, unless that device is
 *    current.
 *  - "stream" is a cudaStream_t passed as void* (NULL = legacy default stream). Calls that
 *    launch work are asynchronous on that stream.
 *  - Device pointers must be 16-byte aligned (KVQ_ERR_ALIGNMENT otherwise); the cache arena
 *    must be 256-byte aligned.
 *  - Ownership: the caller owns every device buffer (cache arena, K/V/q, out, workspace).
 *    The library owns only the small host object returned by kvq_cache_init. It calls no
 *    device allocator.
 *  - Tensors are row-major and contiguous:
 *      K, V  [n_seq, n_kv_heads, n_new, head_dim]   (f32 or bf16)
 *      q     [batch, n_q_heads, head_dim]            (f32 or bf16)
 *      out   [batch, n_q_heads, head_dim]            (f32)
 *    Query head h uses KV head h / (n_q_heads / n_kv_heads) (grouped-query attention).
 *    FP4 (MLA) caches instead take latent [n_seq, n_new, latent_dim] as "K" and the RoPE key
 *    [n_seq, n_new, rope_dim] as "V", the absorbed query q [batch, n_q_heads,
 *    latent_dim + rope_dim] (latent part first) and give out [batch, n_q_heads, latent_dim].
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, inconsistent configuration */
  KVQ_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. head_dim != 128) */
  KVQ_ERR_CAPACITY = 3,     /* append would exceed the cache capacity; nothing written */
  KVQ_ERR_ALIGNMENT = 4,    /* a pointer is not 16-byte (arena: 256-byte) aligned */
  KVQ_ERR_WORKSPACE = 5,    /* workspace or arena smaller than the size query returned */
  KVQ_ERR_CUDA = 6          /* a CUDA launch or copy reported an error */
} kvq_status;

typedef enum {
  KVQ_MODE_LM_QJL = 0,  /* rotation + b-bit Lloyd-Max code + 1-bit QJL residual sketch */
  KVQ_MODE_LM = 1,      /* rotation + b-bit Lloyd-Max code, no sketch */
  KVQ_MODE_SIGN1 = 2,   /* rotation + one sign bit per coordinate (1-bit Lloyd-Max) */
  KVQ_MODE_FP4 = 3,     /* FP4 E2M1 latent, one E4M3 scale per 16 channels (MLA caches) */
  KVQ_MODE_KIVI = 4     /* KIVI-style asymmetric integers, no rotation: keys per channel over groups of 128
                           tokens, values per token (k_mode == v_mode, k_bits == v_bits == 2). The
                           tokens of a sequence's incomplete last key group stay bf16 until it fills */
} kvq_mode;

typedef enum { KVQ_F32 = 0, KVQ_BF16 = 1 } kvq_dtype;

typedef struct {
  int32_t head_dim;     /* LM/SIGN1 modes: 128 */
  int32_t n_q_heads;    /* multiple of n_kv_heads */
  int32_t n_kv_heads;   /* FP4: 1 (one shared latent) */
  int32_t k_mode;       /* kvq_mode; FP4 requires k_mode == v_mode == KVQ_MODE_FP4 */
  int32_t v_mode;
  int32_t k_bits;       /* Lloyd-Max bits for LM modes: 1, 2 or 3 (SIGN1: 1) */
  int32_t v_bits;
  int32_t qjl_dim;      /* sketch rows m; 128 when either side is LM_QJL, else 0 */
  float softmax_scale;  /* 0 => 1/sqrt(dim of q.k): head_dim, or latent_dim + rope_dim */
  int32_t latent_dim;   /* FP4 only: 512 */
  int32_t rope_dim;     /* FP4 only: 64 */
  int32_t rot_per_head; /* LM/SIGN1: 0 = one diagonal D for every KV head; 1 = KV head h has its own
                           D_h (draws h*head_dim .. h*head_dim + head_dim - 1 of rot_seed). FP4: 0 */
  uint64_t rot_seed;    /* seed of the rotation's +-1 diagonal (used when kvq_cache_init gets no
                           rot_signs): see kvq_draw_rotation_signs */
  uint64_t qjl_seed;    /* seed of the sketch matrix S (used when kvq_cache_init gets no qjl_matrix):
                           see kvq_draw_qjl_matrix */
  int32_t sink_tokens;  /* LM/SIGN1 mixed-precision window ("TurboQuant vs OSCAR vs EpiCache", section
                           "Quantization frontiers: TurboQuant and OSCAR": sink and recent tokens stay
                           BF16, the history is quantized): the first sink_tokens tokens of a sequence */
  int32_t recent_tokens;/* and its last recent_tokens tokens are kept as bf16 K and V; the tokens in
                           between are coded as above. 0 and 0 = no window (every token coded).
                           sink_tokens + recent_tokens <= 1024. FP4: both 0 */
} kvq_cfg;

typedef struct kvq_cache kvq_cache; /* opaque host object */

/* The seeded draws, host-only (they fix what kvq_cache_init draws when given no arrays). With the
 * counter-based generator
 *   mix(z)  = z ^= z >> 30; z *= 0xBF58476D1CE4E5B9; z ^= z >> 27; z *= 0x94D049BB133111EB;
 *             z ^= z >> 31                                   (splitmix64 finaliser, mod 2^64)
 *   h(s, i) = mix(s + (i + 1) * 0x9E3779B97F4A7C15)            (draw i of stream s)
 *   U(s, i) = (h(s, i) >> 11) * 2^-53                          (uniform in [0, 1))
 * kvq_draw_rotation_signs writes out[i] = -1 if h(seed, i) is odd, else +1, for i < n.
 * kvq_draw_qjl_matrix writes the row-major [m][d] matrix with entry k = j*d + i equal to the fp32
 * rounding of the Box-Muller normal sqrt(-2 log1p(-U(seed, 2k))) cos(2 pi U(seed, 2k + 1)),
 * computed in double precision with the C library's log1p, sqrt and cos. KVQ_ERR_INVALID_ARG for a
 * null pointer or a non-positive size. */
kvq_status kvq_draw_rotation_signs(uint64_t seed, int32_t n, int8_t* out);
kvq_status kvq_draw_qjl_matrix(uint64_t seed, int32_t m, int32_t d, float* out);

/* Human-readable name of a status code (static string). */
const char* kvq_status_str(kvq_status s);

/* Bytes of device memory a cache of `batch` sequences x `capacity` tokens needs (tables
 * included). capacity is rounded up internally to a multiple of 64 tokens. */
kvq_status kvq_cache_bytes(const kvq_cfg* cfg, int32_t batch, int32_t capacity, size_t* bytes);

/* Packed bytes one token occupies per KV head (codes, sketch and norms of K and V; FP4:
 * latent codes, scales and RoPE key), i.e. the algorithmic bytes decode reads per token. */
kvq_status kvq_packed_bytes_per_token(const kvq_cfg* cfg, size_t* bytes);

/* Create a cache inside caller-owned device memory `dev_mem` (dev_bytes >= kvq_cache_bytes).
 * All sequences start empty. The method's two random draws ("TurboQuant vs OSCAR vs EpiCache",
 * section "Quantization frontiers: TurboQuant and OSCAR": a data-oblivious random rotation, and a
 * Gaussian matrix for the 1-bit QJL sketch) come from the configuration's seeds, or from the
 * caller:
 *   rot_signs: NULL = draw D from cfg->rot_seed (kvq_draw_rotation_signs); else host +1/-1 values,
 *              [head_dim] or, with cfg->rot_per_head, [n_kv_heads][head_dim]. LM/SIGN1 modes only.
 *   qjl_matrix: NULL = draw S from cfg->qjl_seed (kvq_draw_qjl_matrix); else host
 *              [qjl_dim, head_dim] fp32, row-major. Used when a side is LM_QJL.
 * Given arrays are copied; the library keeps no pointer to them after the call returns. The
 * copies into dev_mem are enqueued on `stream`. On success *out owns a host object to free with
 * kvq_cache_destroy. */
kvq_status kvq_cache_init(kvq_cache** out, const kvq_cfg* cfg, int32_t batch, int32_t capacity,
                          void* dev_mem, size_t dev_bytes, const int8_t* rot_signs,
                          const float* qjl_matrix, void* stream);

/* Paged cache ("TurboQuant vs OSCAR vs EpiCache", OSCAR: fused kernels compatible with paged
 * attention and the prefix cache). The tiles of an LM/SIGN1 cache live in a pool of n_pages pages;
 * a page holds 64 consecutive tokens of one sequence for every kv-head (two tiles of K and of V per
 * kv-head). block_table: DEVICE int32 [batch][pages_per_seq], owned by the caller, giving the pool
 * page of each 64-token page of each sequence; capacity = 64 pages_per_seq tokens. The caller fills
 * the entries of the pages a call appends to before the call, and keeps the table unchanged while
 * work that reads it is in flight; sequences may share pages that hold identical tokens (a common
 * prefix) as long as nothing appends into a shared page. The kernels check every entry they use: one
 * that is not a page of the pool (< 0 or >= n_pages) sets KVQ_STATUS_BAD_PAGE; appends then write
 * nothing for that page and decode reads page 0 in its place. kvq_cache_bytes_paged gives the arena
 * size (table excluded); the rest is as for kvq_cache_init. FP4 caches: KVQ_ERR_UNSUPPORTED. */
kvq_status kvq_cache_bytes_paged(const kvq_cfg* cfg, int32_t batch, int32_t n_pages, size_t* bytes);
kvq_status kvq_cache_init_paged(kvq_cache** out, const kvq_cfg* cfg, int32_t batch, int32_t pages_per_seq,
                                int32_t n_pages, const int32_t* block_table, void* dev_mem, size_t dev_bytes,
                                const int8_t* rot_signs, const float* qjl_matrix, void* stream);

/* Quantize n_new tokens per listed sequence and append them ("kvq_quantize(K or V, cfg) ->
 * packed codes + norms + sketch"). K, V: device tensors in the layout above. seq_ids: host
 * array of n_seq distinct sequence indices, or NULL for all sequences in order (then n_seq
 * must equal batch). Fails with KVQ_ERR_CAPACITY, writing nothing, if any listed sequence
 * would exceed the capacity. n_new == 0 or n_seq == 0 is a no-op. The listed sequences are
 * appended by one launch per 1024 of them; KVQ_ERR_CUDA means one of those launches failed: the
 * sequences of the launches before it were appended, and kvq_cache_lengths counts exactly those. */
kvq_status kvq_quantize(kvq_cache* c, const void* K, const void* V, kvq_dtype dtype,
                        int32_t n_new, const int32_t* seq_ids, int32_t n_seq, void* stream);

/* Workspace bytes kvq_decode_attention needs for this cache (split-K partials). */
kvq_status kvq_workspace_bytes(const kvq_cache* c, size_t* bytes);

/* Decode attention of one query per sequence over the packed cache
 * ("kvq_decode_attention(q, packed cache, cfg) -> out"). Every query head attends to all
 * tokens its sequence holds: logits from the codes (plus the QJL correction), softmax in
 * fp32, values dequantised and accumulated on the fly, split over the context with a
 * second-pass combine. A sequence with no tokens gets an all-zero output. */
kvq_status kvq_decode_attention(const kvq_cache* c, const void* q, kvq_dtype dtype, float* out,
                                void* workspace, size_t ws_bytes, void* stream);

/* One decode step: append one token to every sequence (K, V as for kvq_quantize with n_new = 1
 * and all sequences) and run kvq_decode_attention with q over the caches that now include it.
 * The result equals the two calls in sequence; fusing them lets the query prep run while the
 * append is still in flight (on the tensor-core path). Everything is validated (capacity,
 * alignment, workspace for the lengths after the append) before anything is written; a call that
 * fails validation appends nothing. KVQ_ERR_CUDA: if the append's launch failed, nothing was
 * appended and the lengths are unchanged; if a later kernel's launch failed, the append is
 * enqueued and the lengths include it. */
kvq_status kvq_decode_step(kvq_cache* c, const void* K, const void* V, const void* q, kvq_dtype dtype,
                           float* out, void* workspace, size_t ws_bytes, void* stream);

/* Context-parallel decode ("How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2", section
 * "CSA2": the long-context MLA cache; here its context can be split over caches on several GPUs).
 * Each shard -- a cache holding a disjoint part of every sequence's tokens, with the same
 * configuration and seeds -- computes the softmax state of its part, the shards exchange those
 * states (a few KB per sequence, e.g. with an NCCL all-gather), and any of them merges them:
 *   kvq_partial_floats: floats per (sequence, query head) of a state, 2 + dv (dv = head_dim, or
 *     latent_dim for FP4).
 *   kvq_decode_partials: as kvq_decode_attention, but writes partials [batch, n_q_heads, 2 + dv]
 *     (device, f32): m (the largest logit times log2 e), l = sum 2^(logit log2 e - m) and the
 *     unnormalised output o = sum 2^(...) v_hat (in the original, unrotated domain). A sequence with
 *     no tokens gives m = -inf, l = 0, o = 0.
 *   kvq_combine_partials: partials [n_parts][batch, n_q_heads, 2 + dv] (device, contiguous) ->
 *     out [batch, n_q_heads, dv] = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i, M = max_i m_i
 *     (all-zero where every part is empty). Needs no cache; runs on the current device.
 * Merging the states of disjoint shards equals decoding over their union, up to rounding. */
kvq_status kvq_partial_floats(const kvq_cache* c, int32_t* floats);
kvq_status kvq_decode_partials(const kvq_cache* c, const void* q, kvq_dtype dtype, float* partials,
                               void* workspace, size_t ws_bytes, void* stream);
kvq_status kvq_combine_partials(const float* partials, int32_t n_parts, int32_t batch, int32_t n_q_heads,
                                int32_t dv, float* out, void* stream);

/* Device bytes of the staging buffer kvq_decode_step_host needs for inputs of type dtype: two
 * input slots (one step's K and V with n_new = 1 for all sequences, and q), then two output slots;
 * each region 256-byte aligned. */
kvq_status kvq_step_staging_bytes(const kvq_cache* c, kvq_dtype dtype, size_t* bytes);

/* kvq_decode_step with its inputs and output in HOST memory (layouts as for kvq_decode_step;
 * dtype f32 or bf16; out [batch, n_q_heads, head_dim] f32, or latent_dim for FP4). The library
 * keeps two copy streams for the cache (created at the first call, released by
 * kvq_cache_destroy). The copies of K, V and q run on the first, into the input slot of `staging`
 * the step two calls back has finished with, so they overlap the previous step; the step waits
 * for them on `stream`. The copy of out back to host memory runs on the second stream once the
 * step is done, from one of two output slots, so it overlaps the next step. The call returns
 * without waiting. out_event NULL: `stream` also waits for that output copy, and out is valid
 * once `stream` has reached the end of the call's work. out_event a caller-created cudaEvent_t
 * (passed as void*): the library records it after the output copy and `stream` does not wait;
 * out is valid once the event has completed (cudaEventSynchronize, or a stream waiting on it).
 * staging: device, 16-byte aligned, at least
 * kvq_step_staging_bytes, used by nothing else while steps are in flight. Host inputs must be
 * complete when the call is made (not pending writes of GPU work) and unchanged until `stream`
 * has passed the call; pinned (page-locked) memory keeps the copies asynchronous, pageable memory
 * makes the runtime stage them. Everything kvq_decode_step checks is checked before the first
 * copy, so those errors enqueue nothing; KVQ_ERR_CUDA means a copy, event or launch failed,
 * possibly after earlier copies were enqueued. The paper has no counterpart; it keeps a serving
 * loop to one call per step. */
kvq_status kvq_decode_step_host(kvq_cache* c, const void* K, const void* V, const void* q, kvq_dtype dtype,
                                float* out, void* staging, size_t staging_bytes, void* workspace,
                                size_t ws_bytes, void* stream, void* out_event);

/* The same decode attention as kvq_decode_attention, for callers that cannot allocate device
 * memory on the decode path (serving loops that reserve all memory up front, hosts whose memory
 * belongs to another allocator, code that must not risk the device synchronisation cudaMalloc
 * can cause). It takes no workspace and allocates nothing: the split partials go to a fixed
 * 16 MiB device array inside the library, which every GPU that loads the library keeps until
 * the process exits. The paper has no counterpart to this call; it is an interface
 * convenience. Returns KVQ_ERR_WORKSPACE, launching nothing, when the partials of this cache
 * (batch x n_q_heads x splits x (2 + head_dim [+ qjl_dim]) floats; FP4: 2 + latent_dim) would
 * exceed 16 MiB. A call looks up the array's device address on the cache's device (outside stream
 * capture, on every call, so that a device reset and re-created context are followed); a call on
 * a capturing stream reuses the address found by the last uncaptured call on that device, so
 * make the first call on a device before any stream capture (otherwise KVQ_ERR_CUDA). All calls
 * share the array, so calls that overlap on the GPU (different streams, or threads) race: order
 * them on one stream. */
kvq_status kvq_decode_attention_static(const kvq_cache* c, const void* q, kvq_dtype dtype,
                                       float* out, void* stream);

/* Bits of the cache's device status word. The tensor-core decode kernel bounds every wait for
 * staged cache data (about one second of SM clock); a wait that gives up sets
 * KVQ_STATUS_WAIT_TIMEOUT, the kernel still runs to its end and returns, and the output of that
 * call is not to be trusted. KVQ_STATUS_BAD_PAGE: see kvq_cache_init_paged. */
#define KVQ_STATUS_WAIT_TIMEOUT 1
#define KVQ_STATUS_BAD_PAGE 2  /* a paged cache's block table named no page of the pool */

/* Read the cache's device status word (the bits above) into *status (host). Enqueues a 4-byte
 * copy on `stream` and waits for the stream, so it reports on all work enqueued before it.
 * Only kvq_cache_init clears the word. Not part of the method: a failure-detection aid. */
kvq_status kvq_cache_status(const kvq_cache* c, int32_t* status, void* stream);

/* Test entry for the bounded waits (no counterpart in the method): the same call as
 * kvq_decode_attention, except that every CTA of the tensor-core decode kernel first waits on
 * a barrier that nothing ever completes, giving up after wait_limit_cycles SM clock cycles
 * (1 ... 2^31). It then carries on as usual, so the output equals kvq_decode_attention's and
 * KVQ_STATUS_WAIT_TIMEOUT is set. Caches that decode without that kernel (FP4, and LM code
 * combinations it has no instance for) return KVQ_ERR_UNSUPPORTED and launch nothing. */
kvq_status kvq_debug_decode_unset_wait(const kvq_cache* c, const void* q, kvq_dtype dtype, float* out,
                                       void* workspace, size_t ws_bytes, int64_t wait_limit_cycles,
                                       void* stream);

/* Measurement entry (no counterpart in the method): kvq_decode_attention, recording four
 * caller-created CUDA events (cudaEvent_t, passed as void*) on `stream`: events[0] before the
 * first kernel, events[1] after the query prep (right before the split kernel where there is no
 * prep), events[2] after the split kernel, events[3] after the reduce. The events sit between the
 * kernels, so the kernels cannot overlap their neighbours as they do in kvq_decode_attention. */
kvq_status kvq_debug_decode_timed(const kvq_cache* c, const void* q, kvq_dtype dtype, float* out,
                                  void* workspace, size_t ws_bytes, void* stream, void* const* events);

/* Host copy of the current per-sequence lengths (lens: host array of `batch` entries). */
kvq_status kvq_cache_lengths(const kvq_cache* c, int32_t* lens);

/* Byte offsets describing the packed layout, for tools that read the arena directly.
 * info[0..15] receives: tile_tokens, k_tile_bytes, v_tile_bytes, tiles_per_seq,
 * k_region_offset, v_region_offset, then per side (K at 6, V at 11): planes_offset,
 * sketch_offset, norm_offset, gamma_offset, planes; with n_info >= 18 also info[16], info[17]:
 * the order of the K and V planes (0 byte-lane, 1 token, 2 octet); with n_info >= 22 also info[18..21]:
 * the byte offset of the mixed-precision window (bf16 K then V, [batch][n_kv_heads][slots][head_dim]
 * each), slots = sink + recent, sink, recent (zeros without a window). On a window cache the tiles
 * hold the coded history: history token i is sequence position sink + i; with n_info >= 24 also
 * info[22], info[23]: pages_per_seq and n_pages of a paged cache (zeros otherwise: tiles contiguous).
 * Layout of a tile (32 tokens)
 * of one (sequence, kv-head): code bit-planes (512 bytes each), then sign words (512 bytes),
 * then [32] fp16 norms, then [32] fp16 residual norms (sides with a sketch). Plane p holds bit p
 * of every code; a token's 128 bits of a plane are 16 bytes, byte k holding coordinates
 * 8k..8k+7 (coordinate 8k+i in bit i); sign words use the same order (bit = 1 for a
 * non-negative projection). The three orders of those bytes within a plane or the sign block:
 *   byte-lane (values): [16 byte lanes][32 tokens], byte (k, t) = byte k of token t;
 *   token (keys of query groups the tensor-core kernel does not decode): [32 tokens][16 bytes];
 *   octet (all other keys): [4 octets][32 words of 4 bytes], octet o = tokens 8o..8o+7; byte i
 *   of word x = 8t + 2m + h covers coordinate 32m + 16h + 4t + i, bit j of it is token 8o + j.
 * Tiles of a (sequence, kv-head) are consecutive; (sequence, kv-head) pairs follow in row-major
 * order. Capacity is rounded up to whole pairs of tiles (64 tokens).
 * FP4: [32][latent_dim/2] codes (channel 2k in the low nibble of byte k), [32][latent_dim/16]
 * E4M3 scales, [32][rope_dim] bf16 RoPE keys. */
kvq_status kvq_cache_layout(const kvq_cache* c, int64_t* info, int32_t n_info);

/* The fp32 Gaussian Lloyd-Max table the library quantizes against (bits 1..3): centroids
 * [2^bits] ascending, thresholds [2^bits - 1] (midpoints). Host arrays. */
kvq_status kvq_lloyd_max_table(int32_t bits, float* centroids, float* thresholds);

/* Free the host object (the caller still owns and frees the arena). NULL is a no-op. */
void kvq_cache_destroy(kvq_cache* c);

/* Test entry: code already rotated and normalised vectors u [n, head_dim] (device fp32)
 * with the cache's key-side quantizer, writing per vector the code planes
 * [n][k_bits][head_dim/32] u32, the sign words [n][qjl_dim/32] u32 (when the key side has a
 * sketch) and the fp16 residual norm [n] (as uint16 bits). Output pointers are device. */
kvq_status kvq_debug_quantize_rotated(const kvq_cache* c, const float* u, int32_t n,
                                      uint32_t* planes, uint32_t* sketch, uint16_t* gamma,
                                      void* stream);

/* Diagnostic, with no counterpart in the method: the number of GPU kernels this library has
 * enqueued successfully since it was loaded, summed over all threads, devices and caches. A
 * caller reads it before and after a region to learn how many kernels the region launched
 * (quantize: 1 per call; decode: 3 per call on the tensor-core path, else 2). Host-only; never
 * fails. */
uint64_t kvq_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
