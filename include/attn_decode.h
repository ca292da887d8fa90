/*
 * attn_decode.h -- C ABI of libattn_decode.so: single-token decode attention
 * over a paged KV cache on NVIDIA B200 (sm_100a).
 *
 * Sources of the operations (page title, section / equation):
 *   [HEADS] xuesongtap "attention-head" article -- §1 Attention equation
 *           softmax(q K^T / sqrt(d) + M) V with softmax along key positions;
 *           §2 / §2.2 head sharing (MHA H_kv = H_q, GQA contiguous equal
 *           groups of H_q / H_kv, MQA H_kv = 1); §3 causal sliding window
 *           that covers the current position and the w-1 before it, and
 *           whose masked part must be skipped, not computed and masked;
 *           §5.2-§5.3 MLA with U^K absorbed into the query and U^V applied
 *           after the latent-space weighted sum, one softmax over content +
 *           RoPE scores.
 *   [BAIDU] "大模型注意力机制对比：MLA与MQA该怎么选" -- §2 cache shapes
 *           ([batch, heads, seq, head_dim]; MLA [batch, seq, latent + rope])
 *           and §4.3 paged KV-cache management.
 *   [EVOL]  toolsku "注意力機制演進" article -- FlashAttention tiling with
 *           online softmax (the split-KV kernels use that technique).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  * All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees or retains them past the call.  Calls are asynchronous and
 *    ordered on `stream` (a cudaStream_t; NULL = legacy default stream).
 *  * Paged cache: 64-token blocks.  `block_table` is int32 row-major
 *    [B][max_blocks_per_seq]; logical block i of sequence b is physical
 *    block block_table[b * max_blocks_per_seq + i], 0 <= id < num_blocks.
 *    A contiguous (unpaged) cache is the identity table.
 *  * `seq_lens[b]` (int32, device) = T_b tokens cached for sequence b, the
 *    current token included (its K/V is appended before attention); the
 *    query sits at position T_b - 1 and sees keys [lo_b, T_b), where
 *    lo_b = max(0, T_b - window) for window > 0 and 0 otherwise.
 *    T_b = 0 yields a zero output row.
 *  * Host-side validation returns a negative attn_status and launches
 *    nothing.  Faults found on the device (a block id outside
 *    [0, num_blocks), T_b outside [0, 64 * max_blocks_per_seq], a bounded
 *    wait that ran out) never touch memory out of bounds: the offending
 *    sequence/tile is skipped and a per-device error word is set, which
 *    attn_decode_last_error() reports.
 *  * All computation is on the GPU; there is no CPU fallback.
 */
#ifndef ATTN_DECODE_H
#define ATTN_DECODE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ATTN_OK = 0,
    ATTN_ERR_ARG = -1,          /* invalid argument (null, size, alignment) */
    ATTN_ERR_UNSUPPORTED = -2,  /* valid but not implemented (e.g. head dim) */
    ATTN_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed */
    ATTN_ERR_TIMEOUT = -4,      /* device: a bounded wait ran out */
    ATTN_ERR_BAD_BLOCK = -5,    /* device: block id outside [0, num_blocks) */
    ATTN_ERR_BAD_SEQLEN = -6    /* device: T_b < 0, > 64 * max_blocks, or not servable by the ring */
} attn_status;

typedef enum { ATTN_F32 = 0, ATTN_BF16 = 1, ATTN_FP8_E4M3 = 2 } attn_dtype;
/* ATTN_FP8_E4M3 names the cache of attn_decode_gqa_fp8 in
 * attn_decode_gqa_config only; the decode entry points take F32 or BF16. */

/* Tokens per cache block (fixed by the storage format). */
#define ATTN_BLOCK_SIZE 64

/*
 * attn_decode_gqa -- decode attention for MHA / GQA / MQA ([HEADS] §1, §2).
 *
 *   out[b,h,:] = sum_{j in [lo_b, T_b)} softmax_j(scale * <q[b,h], K[b,g(h),j]>)
 *                 * V[b,g(h),j,:],     g(h) = floor(h / (H_q / H_kv))
 *
 * q        [B][H_q][d]                   dtype, contiguous
 * k_cache  [num_blocks][H_kv][64][d]     dtype; one (block, head) tile is
 * v_cache  [num_blocks][H_kv][64][d]     64*d contiguous elements
 * out      [B][H_q][d]                   dtype (rounded to nearest even)
 * window   > 0: causal sliding window of that many positions, the current one
 *          included ([HEADS] §3); <= 0: full causal.  Blocks wholly outside
 *          the window are never read.
 * dtype    ATTN_BF16 (any supported d) or ATTN_F32 (d <= 128); accumulation
 *          is always fp32.
 * Requirements: H_q % H_kv == 0; d in {16, 32, 64, 128, 256}; pointers
 * 16-byte aligned; B >= 1; max_blocks_per_seq >= 1; num_blocks >= 1.
 * Uses a library-owned split workspace (partials and arrival counters) per
 * device and stream, so calls on different streams may run at the same time.
 * A stream's workspace is grown (cudaMalloc) on first use outside stream
 * capture; growing it while the stream is being captured returns
 * ATTN_ERR_UNSUPPORTED.  Up to 16 streams per device keep their own; another
 * stream takes over the least recently used one's (after a cudaFree, which
 * waits for the device).  The per-thread default stream is keyed by the
 * calling thread.  The device error word read by attn_decode_last_error is
 * shared by all streams of the device.
 */
int attn_decode_gqa(const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *seq_lens, const int32_t *block_table,
                    void *out, int B, int H_q, int H_kv, int d, float scale,
                    int window, void *stream, int max_blocks_per_seq,
                    int num_blocks, int dtype);

/*
 * attn_decode_mla -- absorbed MLA decode ([HEADS] §5.2, §5.3).
 *
 *   s_j     = scale * (<q_latent[b,h], c_j> + <q_rope[b,h], kR_j>)
 *   out[b,h,:] = sum_{j < T_b} softmax_j(s) * c_j          (d_c wide)
 *
 * q_latent     [B][H][d_c]  bf16  absorbed query q^C (U^K_h)^T
 * q_rope       [B][H][d_r]  bf16  rotated RoPE query
 * latent_cache [num_blocks][64][d_c + d_r] bf16: row = c_j followed by the
 *              already-rotated shared RoPE key kR_j
 * out          [B][H][d_c]  bf16  latent-space output z (apply U^V_h after)
 * Supported: d_c = 512, d_r = 64, H = 128 (the tensor-core tile is 128
 * heads); otherwise ATTN_ERR_UNSUPPORTED.  Workspace as for attn_decode_gqa.
 * Runs as clusters of two CTAs; uses 512 TMEM columns per CTA.
 */
int attn_decode_mla(const void *q_latent, const void *q_rope,
                    const void *latent_cache, const int32_t *seq_lens,
                    const int32_t *block_table, void *out, int B, int H,
                    int d_c, int d_r, float scale, void *stream,
                    int max_blocks_per_seq, int num_blocks);

/*
 * kv_append -- write the new token's K and V of every sequence into its
 * paged slot ([BAIDU] §4.3 paging; [EVOL] cache concatenation before
 * attention).  Position positions[b] (usually T_b - 1) lands in logical block
 * positions[b] / 64, row positions[b] % 64, for every KV head.
 * k_new, v_new [B][H_kv][d] dtype; caches as in attn_decode_gqa.
 * Rows whose position or block id is out of range are skipped and flagged
 * (ATTN_ERR_BAD_BLOCK).  Pointers 16-byte aligned; d as above.
 */
int kv_append(const void *k_new, const void *v_new, void *k_cache,
              void *v_cache, const int32_t *positions,
              const int32_t *block_table, int B, int H_kv, int d,
              int max_blocks_per_seq, int num_blocks, int dtype,
              void *stream);

/*
 * kv_append_mla -- write each sequence's new latent row (c followed by kR,
 * d_c + d_r bf16 values) into latent_cache at positions[b].
 * latent_new [B][d_c + d_r] bf16.  (d_c + d_r) * 2 must be a multiple of 16.
 */
int kv_append_mla(const void *latent_new, void *latent_cache,
                  const int32_t *positions, const int32_t *block_table,
                  int B, int d_c, int d_r, int max_blocks_per_seq,
                  int num_blocks, void *stream);

/*
 * attn_visibility -- which cached keys each query sees, and how the block
 * table row maps them (attention-head article, §3 sliding window; window plus
 * global tokens G).  Key j of a sequence with T = seq_lens[b] cached tokens is
 * visible to the decode query (position T - 1) when j < T and (window <= 0,
 * or j >= T - window, or j < sink_tokens, or j is a global position of the
 * sequence, or T - 1 is itself a global position: a global query sees the
 * whole history).  Global positions: global_pos is a device int32 array
 * [B][n_global], row b holding sequence b's positions in ascending order;
 * the row ends at its first entry that does not exceed the previous one (pad
 * with -1).  0 < n_global <= 64; global_pos needs sink_tokens = 0
 * (ATTN_ERR_ARG otherwise; n_global > 64: ATTN_ERR_UNSUPPORTED);
 * n_global = 0 ignores global_pos.  Blocks before the window hold visible
 * keys only where a global position lies, and only those blocks are read.
 * ring_blocks > 0 makes the table row a ring for window layers: the blocks
 * holding the sink keys keep slots [0, A) with A = ceil(sink_tokens / 64),
 * and logical block i >= A lives in slot A + (i mod ring_blocks), so a
 * sequence stores only the blocks its window can reach; kv_append_ext
 * writing token T-1 then overwrites (evicts) the block that left the
 * window.  With a global set, the row instead starts with A = n_global
 * global slots: slot k names the block holding position global_pos[b][k]
 * (slots of positions that share a block name the same block; slots after
 * the row's end are not read), a block before the window's first block
 * (logical block max(0, T - window) / 64) is read through the global slot
 * of its first global position, and logical block i from the window's first
 * block on lives in slot A + (i mod ring_blocks).  The caller keeps a global
 * position's block alive in its global slot when the ring moves past it
 * (gives the ring slot a new block); kv_append_ext with the same record
 * writes through the ring slots.  A global query (T - 1 a global position)
 * with T > window would need keys the ring no longer holds: that sequence
 * is refused on the device (ATTN_ERR_BAD_SEQLEN from attn_decode_last_error,
 * zero output row).  ring_blocks > 0 requires window > 0, ring_blocks * 64 >=
 * window + 63 (the ring holds every block a window can touch) and
 * A + ring_blocks <= max_blocks_per_seq; T is then not limited by the table
 * width.  All zero: full causal attention, identity table (attn_decode_gqa).
 */
typedef struct attn_visibility {
    int window;
    int sink_tokens;
    int ring_blocks;
    const int32_t *global_pos;   /* device, [B][n_global]; may be NULL if n_global == 0 */
    int n_global;
} attn_visibility;

/*
 * attn_decode_gqa_ext -- attn_decode_gqa with global (sink) tokens and a
 * ring-buffer table (see attn_visibility; visibility must be non-null, host
 * memory, read during the call).  Blocks holding no visible key are never
 * read.  Same arguments, layouts, workspace and errors as attn_decode_gqa,
 * plus ATTN_ERR_ARG for an invalid visibility record.
 */
int attn_decode_gqa_ext(const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *seq_lens, const int32_t *block_table, void *out,
                        int B, int H_q, int H_kv, int d, float scale,
                        const attn_visibility *visibility, void *stream,
                        int max_blocks_per_seq, int num_blocks, int dtype);

/*
 * kv_append_ext -- kv_append through the table mapping of `visibility`
 * (sink slots, then the ring): token positions[b] goes to offset
 * positions[b] % 64 of the block in slot table_slot(positions[b] / 64).
 * A slot outside the table row or a block id outside the pool sets the
 * bad-block error bit and skips that row.
 */
int kv_append_ext(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                  const int32_t *positions, const int32_t *block_table, int B, int H_kv,
                  int d, int max_blocks_per_seq, int num_blocks, int dtype,
                  const attn_visibility *visibility, void *stream);

/*
 * attn_decode_plan -- run the device split planner on its own and write the
 * plan the decode kernels would follow (for bit-exact checks against a host
 * model).  The flattened work list orders sequences b, then units
 * (unit = a KV head, or a chunk of its query heads) of that sequence, then
 * the visible 64-token blocks of the unit.  CTA i of num_ctas takes blocks
 * [floor(i*W/num_ctas), floor((i+1)*W/num_ctas)) of the W in total.
 * Output (int64, device) plan_out: [0] = W, then for every CTA i four
 * values: range start, range end, sequence of the first block, unit of the
 * first block (-1, -1 for an empty range); then B+1 exclusive prefix sums
 * of blocks per sequence.  Size: 1 + 4*num_ctas + B + 1 int64.
 * units_per_seq = H_kv * (query-head chunks per KV head).
 */
int attn_decode_plan(const int32_t *seq_lens, int B, int units_per_seq,
                     int window, int max_blocks_per_seq, int num_ctas,
                     int64_t *plan_out, void *stream);

/*
 * attn_decode_gqa_config -- the launch shape attn_decode_gqa uses for a
 * problem: *num_ctas = CTAs of the split-KV kernel, *heads_per_cta = query
 * heads a CTA processes per KV head (the group is split into
 * H_q / H_kv / heads_per_cta chunks when it does not fit), *path = 0 for the
 * CUDA-core kernel, 1 for the M = 128 tensor-core (tcgen05) kernel, 2 for
 * the M = 64 tensor-core kernel.  dtype ATTN_FP8_E4M3 answers for
 * attn_decode_gqa_fp8.
 */
int attn_decode_gqa_config(int B, int H_q, int H_kv, int d, int dtype,
                           int *num_ctas, int *heads_per_cta, int *path);

/*
 * attn_set_num_ctas -- testing/tuning hook: force the number of split-KV CTAs
 * used by later calls on this host thread's current device (0 = automatic).
 */
int attn_set_num_ctas(int num_ctas);

/*
 * attn_set_gqa_path -- testing/tuning hook: -1 = automatic (bf16: the
 * CUDA-core kernel for groups of up to 4 heads, the tensor-core path for
 * larger groups; fp8 cache: the M = 128 tensor-core kernel for d <= 128 and
 * groups of 16 to 32 heads or multiples of 32, else the CUDA-core kernel),
 * 0 = force the CUDA-core kernel, 1 = force the tensor-core path (the M = 128
 * kernel where it applies, d <= 128 and units of <= 32 heads, else the M = 64
 * kernel, which has no fp8 form), 2 = force the M = 64 tensor-core kernel
 * (fp8 calls then run on the CUDA cores).
 */
int attn_set_gqa_path(int path);

/*
 * attn_set_profile_events -- optional timing hook.  When n > 0, the next n
 * decode calls record start_events[i] / stop_events[i] (cudaEvent_t handles
 * owned by the caller) on their stream immediately around their main split-KV
 * kernel; n = 0 disables.  The arrays must stay valid until disabled.
 */
int attn_set_profile_events(void *const *start_events,
                            void *const *stop_events, int n);

/*
 * attn_debug_force_timeout -- fault-injection hook for tests: when enable is
 * nonzero, the next decode launch waits on a barrier that is never signalled,
 * bounded by timeout_ns, then sets ATTN_ERR_TIMEOUT and returns without
 * hanging the device.  One-shot.
 */
int attn_debug_force_timeout(int enable, long long timeout_ns);

/*
 * attn_decode_last_error -- synchronise `stream`, then read and clear the
 * current device's error word.  Returns ATTN_OK, or the first device-side
 * status (ATTN_ERR_TIMEOUT, ATTN_ERR_BAD_BLOCK, ATTN_ERR_BAD_SEQLEN), or
 * ATTN_ERR_CUDA if the synchronisation itself failed.
 */
int attn_decode_last_error(void *stream);

/*
 * attn_decode_gqa_noalloc -- attn_decode_gqa for callers that may not
 * allocate device memory while they run.  (The source pages have no
 * counterpart: this is a deployment variant of the same operation.)
 *
 * Some callers cannot call cudaMalloc/cudaFree after start-up: a serving
 * process that gives all device memory to its own pool, or a latency-critical
 * thread that cannot take the device-wide synchronisation cudaFree implies.
 * This entry point computes the same operation as attn_decode_gqa, with the
 * same arguments and layouts, always on the CUDA-core split kernel (so it
 * agrees with attn_decode_gqa within the parity tolerance, not bit for bit
 * where that call picks a tensor-core kernel), but keeps its split scratch
 * in a fixed array
 * of ATTN_NOALLOC_SCRATCH_BYTES compiled into the library (every GPU that
 * loads the library holds that array until the process exits).  It never
 * allocates.  The caller still passes all inputs and the output.
 *
 * Scratch needed: 4 * (B*H_q/hc + SMs) * hc * (d + 1) bytes plus 8*(B+1)
 * (hc = query heads per CTA, see attn_decode_gqa_config; each term rounded
 * up to 256 bytes), and at most ATTN_NOALLOC_MAX_UNITS (sequence, KV head,
 * head chunk) units, B*H_q/hc; above either limit the call returns
 * ATTN_ERR_UNSUPPORTED.  A second fixed array holds one split-arrival
 * counter per unit: zero when the library loads, zero again after every
 * call.  The first call on each device looks up the arrays' device
 * addresses (cudaGetSymbolAddress, on the current device); make that first
 * call before any stream capture.  All calls share the arrays and the
 * scratch keeps the last call's contents (nothing in it needs to start at
 * zero): calls that can overlap on the GPU -- on different streams, or from
 * several threads -- race on them, so order them on one stream.  The attn_set_num_ctas, profiling and
 * fault-injection hooks do not apply to this entry point.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (8u << 20)
#define ATTN_NOALLOC_MAX_UNITS 65536
int attn_decode_gqa_noalloc(const void *q, const void *k_cache,
                            const void *v_cache, const int32_t *seq_lens,
                            const int32_t *block_table, void *out, int B,
                            int H_q, int H_kv, int d, float scale, int window,
                            void *stream, int max_blocks_per_seq,
                            int num_blocks, int dtype);

/*
 * attn_decode_gqa_fp8 -- attn_decode_gqa over an fp8 KV cache: quantised
 * K/V halve the bytes the bandwidth-bound decode reads.  k_cache / v_cache
 * [num_blocks][H_kv][64][d] hold OCP FP8 E4M3 codes (1 byte); k_scale /
 * v_scale [num_blocks][H_kv][64] fp32 hold one scale per cached row, so the
 * key/value used is code_value * row_scale (as written by kv_append_fp8).
 * q and out are bf16 [B][H_q][d]; d in {64, 128, 256}; every group size runs
 * on the CUDA-core kernel.  visibility may be null (full causal, identity
 * table) or as for attn_decode_gqa_ext.  Scale arrays 16-byte aligned; other
 * arguments, workspace and errors as attn_decode_gqa.
 */
int attn_decode_gqa_fp8(const void *q, const void *k_cache, const void *v_cache,
                        const float *k_scale, const float *v_scale, const int32_t *seq_lens,
                        const int32_t *block_table, void *out, int B, int H_q, int H_kv, int d,
                        float scale, const attn_visibility *visibility, void *stream,
                        int max_blocks_per_seq, int num_blocks);

/*
 * kv_append_fp8 -- quantise and append the current token's K and V rows
 * (bf16 [B][H_kv][d]) into the fp8 cache at positions[b] (through the table
 * mapping of `visibility`, which may be null).  Each row x of d values is
 * stored as E4M3 codes of x * (448 / amax), rounded to nearest even and
 * saturated to +-448, with row scale amax / 448 (amax = max |x| in fp32; a
 * zero row gets scale 0 and zero codes); both divisions are IEEE
 * round-to-nearest.  Errors as kv_append.
 */
int kv_append_fp8(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                  float *k_scale, float *v_scale, const int32_t *positions,
                  const int32_t *block_table, int B, int H_kv, int d, int max_blocks_per_seq,
                  int num_blocks, const attn_visibility *visibility, void *stream);

/*
 * attn_decode_mla_fp8 -- attn_decode_mla over an fp8 latent cache: the
 * shared latent rows (the cache MLA keeps, attention-head §5.4) stored as
 * OCP FP8 E4M3 codes, halving the bytes a decode streams ([BAIDU] §4.3: the
 * cache-quantisation schemes a serving stack carries).
 * latent_codes [num_blocks][64][d_c + d_r] uint8 E4M3 codes; latent_scale
 * [num_blocks][64] fp32, one scale per cached row, so c_j / kR_j are the code
 * values times the row scale (as written by kv_append_mla_fp8).  q_latent,
 * q_rope and out are bf16 as for attn_decode_mla; d_c = 512, d_r = 64,
 * H = 128.  The codes are widened to bf16 exactly on the chip; NaN codes
 * (S.1111.111, never written by kv_append_mla_fp8) read as +-480.
 * latent_scale 16-byte aligned; other arguments, workspace and errors as
 * attn_decode_mla.
 */
int attn_decode_mla_fp8(const void *q_latent, const void *q_rope, const void *latent_codes,
                        const float *latent_scale, const int32_t *seq_lens,
                        const int32_t *block_table, void *out, int B, int H, int d_c, int d_r,
                        float scale, void *stream, int max_blocks_per_seq, int num_blocks);

/*
 * kv_append_mla_fp8 -- quantise and append each sequence's new latent row
 * (latent_new [B][d_c + d_r] bf16, c followed by kR) into the fp8 latent cache
 * at positions[b]: codes of x * (448 / amax), rounded to nearest even and
 * saturated to +-448, with row scale amax / 448 (amax = max |x| over the whole
 * row, fp32; a zero row gets scale 0 and zero codes; both divisions IEEE
 * round-to-nearest), exactly as kv_append_fp8 quantises a K/V row.
 * latent_codes / latent_scale as for attn_decode_mla_fp8.  d_c + d_r even;
 * latent_new and latent_codes 16-byte aligned.  Errors as kv_append.
 */
int kv_append_mla_fp8(const void *latent_new, void *latent_codes, float *latent_scale,
                      const int32_t *positions, const int32_t *block_table, int B, int d_c,
                      int d_r, int max_blocks_per_seq, int num_blocks, void *stream);

/*
 * attn_mla_absorb_q -- the key up-projection folded into the query, before
 * the absorbed MLA decode (attention-head §5.2): per sequence b and head h,
 *     q_latent[b][h][:] = sum_i q_c[b][h][i] * u_k[h][:][i]
 * i.e. q_c (U^K_h)^T with k^C_j = c_j U^K_h.  q_c [B][H][d_h], u_k
 * [H][d_c][d_h], q_latent [B][H][d_c] (the q_latent input of
 * attn_decode_mla); all bf16, device, 16-byte aligned, row-major; fp32
 * accumulation, result rounded to bf16 (nearest even).  d_c a multiple of
 * 128 and d_h a multiple of 64, H <= 65535 (ATTN_ERR_UNSUPPORTED otherwise).
 * Stream-ordered; a tcgen05 tensor-core kernel that reads each head's weight
 * once per call and reuses it for all B sequences.  Allocates nothing.
 */
int attn_mla_absorb_q(const void *q_c, const void *u_k, void *q_latent, int B, int H,
                      int d_c, int d_h, void *stream);

/*
 * attn_mla_project_out -- the value up-projection after the absorbed MLA
 * decode (attention-head §5.2): per sequence b and head h,
 *     o[b][h][:] = sum_c z[b][h][c] * u_v[h][c][:]
 * i.e. z U^V_h with v_j = c_j U^V_h.  z [B][H][d_c] (the output of
 * attn_decode_mla), u_v [H][d_c][d_v], o [B][H][d_v]; bf16, device, 16-byte
 * aligned, row-major; fp32 accumulation, result rounded to bf16 (nearest
 * even).  d_v a multiple of 128 and d_c a multiple of 64, H <= 65535
 * (ATTN_ERR_UNSUPPORTED otherwise).  Stream-ordered; the same tensor-core
 * kernel as attn_mla_absorb_q, U^V_h read once per call.  Allocates nothing.
 */
int attn_mla_project_out(const void *z, const void *u_v, void *o, int B, int H, int d_c,
                         int d_v, void *stream);

/* Human-readable name of a status code (static storage). */
const char *attn_status_string(int status);

/* Library version: major * 10000 + minor * 100 + patch. */
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_DECODE_H */
