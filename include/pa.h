/*
 * pa.h — C ABI of libpa: paged KV-cache append and paged decode attention
 * for NVIDIA B200 (sm_100a), plus the host-side block manager that feeds them.
 *
 * Every entry point takes plain pointers and sizes.  Device pointers are
 * CUDA device addresses owned by the caller; the library never allocates,
 * frees or keeps device memory, and never synchronises unless a function says
 * so.  `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 * stream); work is enqueued on it asynchronously.  Functions return a status
 * code (PA_OK or a negative PA_ERR_*); no C++ exception crosses this ABI.
 *
 * bf16 tensors are passed as pa_bf16 (the raw 16-bit pattern: sign, 8-bit
 * exponent, 7-bit mantissa — the upper half of an IEEE-754 float, as the
 * Tiny-vLLM summary page "[Hacker News 요약] ... Tiny-vLLM ..." (aisleshub)
 * describes bfloat16 in its section "모델 로딩 및 데이터 형식 심층 이해").
 *
 * Where the operations come from:
 *  - Paging: page "vLLM — PagedAttention으로 LLM 추론 성능을 2~4배 끌어올린 서빙
 *    엔진" (dev.to), section "PagedAttention — OS 가상 메모리에서 영감": the KV
 *    cache is divided into fixed-size blocks handed out only as tokens arrive,
 *    and logical blocks are mapped to non-contiguous physical blocks.
 *  - KV cache and attention: same page, section "KV Cache가 왜 병목인가", and
 *    the Tiny-vLLM summary page, section "고성능 추론을 위한 고급 최적화 기법":
 *    K/V of earlier tokens are stored and re-read at every decode step;
 *    attention is softmax(q K^T * scale) V; grouped-query attention lets
 *    several query heads share one K/V head; the causal mask lets the decode
 *    query (the newest position) see every cached token.
 *  - Block manager: page "Nano-vLLM로 배우는 vLLM 추론 엔진 작동 원리 한눈에
 *    정리" (tilnote.io), section "KV 캐시와 Block Manager": fixed-size blocks,
 *    metadata on the CPU, K/V tensors on the GPU, shared prefix blocks.
 *  - Decode is memory-bound (dev.to page, section "Prefill vs Decode"), which
 *    is why the decode kernel streams each K/V page from HBM once per kv head
 *    and splits long contexts across CTAs.
 *
 * Layouts (all row-major, contiguous):
 *   k_cache, v_cache  [num_blocks][num_kv_heads][block_size][head_dim] bf16
 *   q, out            [num_seqs][num_q_heads][head_dim]               bf16
 *   k, v (append)     [num_tokens][num_kv_heads][head_dim]            bf16
 *   slot_mapping      [num_tokens] int64: slot = block * block_size + offset
 *   block_tables      [num_seqs][max_blocks_per_seq] int32: physical block of
 *                     logical block i; entries past a sequence's last block
 *                     are never read
 *   context_lens      [num_seqs] int32: tokens the decode query attends to,
 *                     the token appended this step included
 * Query head h reads kv head h / (num_q_heads / num_kv_heads).
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

typedef uint16_t pa_bf16;

/* ---- status codes ---------------------------------------------------------------------- */
#define PA_OK                 0
#define PA_ERR_INVALID       -1  /* null pointer, bad size, misaligned pointer, Hq % Hkv != 0 */
#define PA_ERR_UNSUPPORTED   -2  /* well-formed but outside the built shapes (see pa_decode) */
#define PA_ERR_CUDA          -3  /* a CUDA runtime call or kernel launch failed */
#define PA_ERR_WORKSPACE     -4  /* workspace missing, misaligned or smaller than required */
#define PA_ERR_OOM_BLOCKS    -5  /* block manager: not enough free blocks */
#define PA_ERR_SHARED_BLOCK  -6  /* block manager: append into a block that several tables hold */
#define PA_ERR_BAD_BLOCK     -7  /* decode saw a block id outside [0, num_blocks) */
#define PA_ERR_BAD_LENGTH    -8  /* decode saw a context length above max_context_len or the table */
#define PA_ERR_TIMEOUT       -9  /* a bounded wait inside a kernel gave up */

/* Human-readable name of a status code (static string, never NULL). */
PA_API const char* pa_status_string(int status);

/* ---- pool geometry ---------------------------------------------------------------------- */
typedef struct pa_cache_desc {
    int32_t num_blocks;          /* N: physical blocks in each cache tensor                   */
    int32_t block_size;          /* Bs: tokens per block                                       */
    int32_t num_kv_heads;        /* Hkv                                                        */
    int32_t num_q_heads;         /* Hq, a multiple of Hkv                                      */
    int32_t head_dim;            /* D                                                          */
    int32_t max_blocks_per_seq;  /* MB: row stride of block_tables                             */
} pa_cache_desc;

/* ---- KV append ------------------------------------------------------------------------- */
/*
 * Writes token t's K and V rows (all kv heads) into slot slot_mapping[t] of
 * k_cache / v_cache: block s / Bs, offset s % Bs.  A negative slot, or one
 * at or past num_blocks * block_size, writes nothing.  The copy is bit-exact;
 * no other byte of the caches changes.  Two tokens mapped to the same slot
 * race (the survivor is unspecified).
 * Requirements: head_dim a multiple of 8; k, v, k_cache, v_cache 16-byte
 * aligned.  num_tokens == 0 is a no-op.
 * Errors: PA_ERR_INVALID (arguments), PA_ERR_CUDA (launch).
 */
PA_API int pa_append_kv(const pa_bf16* k, const pa_bf16* v, const int64_t* slot_mapping,
                 int32_t num_tokens, pa_bf16* k_cache, pa_bf16* v_cache,
                 const pa_cache_desc* desc, void* stream);

/*
 * FP8 KV append.  The Tiny-vLLM summary page ("[Hacker News 요약] ... Tiny-vLLM
 * ...", section "향후 전망") names FP8 among the data types to add, with no format
 * or scale scheme.  This library uses the OCP E4M3 format (1 sign, 4 exponent
 * bits of bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN, largest
 * finite 448) with one scale per cache tensor: a bf16 value x is stored as the
 * code of float(x) * float(1/scale) (one float multiply) rounded to nearest
 * even, saturating at +-448, and reads back as code value * scale.  Halves the
 * bytes every decode reads.
 * Same slots and requirements as pa_append_kv; k_cache / v_cache are uint8
 * pools [N][Hkv][Bs][D] (8-byte aligned); k_scale, v_scale > 0 and finite.
 */
PA_API int pa_append_kv_e4m3(const pa_bf16* k, const pa_bf16* v, const int64_t* slot_mapping,
                             int32_t num_tokens, float k_scale, float v_scale, uint8_t* k_cache,
                             uint8_t* v_cache, const pa_cache_desc* desc, void* stream);

/*
 * RoPE (rotary position embedding) fused with the KV append.  The Tiny-vLLM
 * summary page ("[Hacker News 요약] ... Tiny-vLLM ...", section "핵심 LLM 연산의
 * CUDA 커널 구현") names RoPE among the per-layer kernels of the model it
 * targets, without a formula; this library applies RoFormer's rotation in the
 * rotate-half pairing: for i < D/2 the pair (x[i], x[i + D/2]) of every head of
 * token t turns by the angle positions[t] * rope_theta^(-2i/D):
 *   y[i] = x[i] cos a - x[i + D/2] sin a,   y[i + D/2] = x[i] sin a + x[i + D/2] cos a.
 * Angles are formed in double, cos/sin and the rotation in float, and every
 * rotated row is rounded to nearest-even bf16.
 *
 * q: [num_tokens][Hq][D] bf16, rotated into q_out (q_out == q rotates in
 * place).  k: [num_tokens][Hkv][D] bf16, rotated and written into slot
 * slot_mapping[t] of k_cache; v: the same shape, copied unchanged into the
 * same slot of v_cache.  Slots follow pa_append_kv (negative or past the pool:
 * nothing written for that token's K/V; its q is still rotated).  positions:
 * [num_tokens] int32 device array.  rope_theta > 0.
 * Requirements: head_dim 64 or 128; q, q_out, k, v, k_cache, v_cache 16-byte
 * aligned.  num_tokens == 0 is a no-op.
 * Errors: PA_ERR_INVALID (arguments), PA_ERR_UNSUPPORTED (head_dim), PA_ERR_CUDA.
 */
PA_API int pa_rope_append_kv(const pa_bf16* q, pa_bf16* q_out, const pa_bf16* k, const pa_bf16* v,
                             const int32_t* positions, const int64_t* slot_mapping,
                             int32_t num_tokens, float rope_theta, pa_bf16* k_cache,
                             pa_bf16* v_cache, const pa_cache_desc* desc, void* stream);

/* ---- paged decode attention ------------------------------------------------------------ */
#define PA_KERNEL_AUTO          0  /* the fastest built kernel for the shape                    */
#define PA_KERNEL_SIMT          1  /* CUDA cores: plain loads, fp32 FMA                         */
#define PA_KERNEL_TENSOR        2  /* tensor cores (mma.sync bf16), TMA-staged pages; whole kv-  */
                                   /* head groups of 8 per CTA when Hkv % 8 == 0, else per head */
#define PA_KERNEL_TENSOR_SPLIT  3  /* tensor cores, one (sequence, kv head, split) per work item */

#define PA_FLAG_CHECK     1   /* synchronise after the launch and report device-side errors     */
#define PA_FLAG_PDL       2   /* early start (programmatic dependent launch), see pa_decode     */
/* Failure-handling self-test (whole-group tensor kernel only, else PA_ERR_UNSUPPORTED): the
 * producer warp of the kernel's CTA 0 issues no copy and signals nothing, so that CTA's
 * consumer warps find their first wait unanswered; their waits give up after 10 ms (instead
 * of 2 s), raise the timeout bit and the CTA exits with no copy in flight.  The other CTAs run
 * normally.  The call then reports PA_ERR_TIMEOUT (through PA_FLAG_CHECK or pa_decode_status)
 * and its output is unspecified; the workspace serves the next call as it is.  For tests of
 * the error path; never set in normal use. */
#define PA_FLAG_SELFTEST_STALL 4

#define PA_KV_BF16        0   /* caches hold bf16 values                                         */
#define PA_KV_E4M3        1   /* caches hold E4M3 codes (uint8), see pa_append_kv_e4m3           */

typedef struct pa_decode_options {
    int32_t split_tokens;  /* SIMT / TENSOR_SPLIT: 0 automatic, else tokens per KV split, a      */
                           /* positive multiple of 64                                           */
    int32_t kernel;        /* PA_KERNEL_*                                                        */
    int32_t flags;         /* PA_FLAG_*                                                          */
    int32_t max_ctas;      /* TENSOR: 0 = one CTA per resident slot, else at most this many      */
    float rope_theta;      /* pa_append_decode only: > 0 turns q and the new K rows by RoPE at   */
                           /* position L-1 with this frequency base (see pa_rope_append_kv);    */
                           /* 0 = no rotation.  pa_decode(_ex) rejects a nonzero value.         */
    int32_t kv_dtype;      /* PA_KV_BF16 (default) or PA_KV_E4M3: the caches are uint8 E4M3     */
                           /* pools of the same [N][Hkv][Bs][D] shape (the pointers are read as */
                           /* bytes); the whole-group tensor kernel only                        */
    float k_scale;         /* PA_KV_E4M3: K value = code value * k_scale (> 0)                  */
    float v_scale;         /* PA_KV_E4M3: V value = code value * v_scale (> 0)                  */
} pa_decode_options;

/*
 * Bytes of device workspace pa_decode needs for this batch shape (0 on bad
 * arguments).  max_context_len is an upper bound of every context_lens[b].
 * Needs a current CUDA device (the split plan depends on its SM count).
 */
PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t max_context_len,
                                const pa_cache_desc* desc);
PA_API size_t pa_decode_workspace_size_ex(int32_t num_seqs, int32_t max_context_len,
                                   const pa_cache_desc* desc, const pa_decode_options* options);

/*
 * Paged decode attention: for every sequence b and query head h,
 *   out[b][h] = bf16( sum_j p_j V_j ),  p = softmax_j(scale * q[b][h] . K_j),
 * over the context_lens[b] tokens the table row block_tables[b] reaches,
 * with K_j, V_j the rows of kv head h / (Hq/Hkv).  fp32 accumulation, online
 * softmax, the result rounded to nearest-even bf16.  A sequence with
 * context_lens[b] == 0 outputs zeros.  Long contexts are split across CTAs:
 * each piece leaves an fp32 partial state in the workspace, and a second
 * kernel, launched by the same call on the same stream, merges them
 * (log-sum-exp) into out.
 *
 * workspace: caller-owned device buffer of at least
 * pa_decode_workspace_size(...) bytes, 256-byte aligned, ZERO-FILLED BEFORE
 * ITS FIRST USE.  The kernels leave their work counters at zero when they
 * complete, so the buffer can be reused by later calls without clearing;
 * calls that may overlap on the GPU need separate workspaces.
 *
 * Built shapes: head_dim 64 or 128; block_size 8, 16, 32, 64, 128 or 256;
 * Hq / Hkv <= 16.  Others return PA_ERR_UNSUPPORTED.  The tensor-core
 * kernels need the CUDA driver's tensor-map encoder; an explicit
 * PA_KERNEL_TENSOR(_SPLIT) request that cannot be served returns
 * PA_ERR_UNSUPPORTED (no silent fallback).  Pointers q, out,
 * k_cache, v_cache must be 16-byte aligned.
 * A block id outside [0, num_blocks) is read as zeros and a length above
 * max_context_len or the table is clipped; both raise a bit in the
 * workspace's status word, which pa_decode_status reports (PA_FLAG_CHECK
 * does so before returning).
 *
 * options->kv_dtype == PA_KV_E4M3: the caches are E4M3 pools (see
 * pa_append_kv_e4m3) and the attention reads K = code value * k_scale,
 * V = code value * v_scale; only the whole-group tensor kernel serves it
 * (PA_ERR_UNSUPPORTED otherwise).  pa_append_decode then quantizes the new
 * rows with the same scales as it writes them; with rope_theta > 0 the new K
 * row is turned and rounded to bf16 first, and that bf16 row is quantized.
 *
 * PA_FLAG_PDL (whole-group tensor kernel only; ignored by the others): the
 * decode kernel is launched as a programmatic dependent of the kernel before
 * it on `stream`, so it may start while that kernel is still running.  Before
 * it waits for that kernel to complete it reads ONLY context_lens and
 * block_tables (to plan its slice of the work); q, the caches, out and the
 * workspace are touched after the wait.  Set the flag only when context_lens
 * and block_tables were complete before the previous kernel on `stream`
 * started (host-written metadata, as in a serving step's layer loop).  The
 * library's own kernels (append, merge) let such a launch start early.
 */
PA_API int pa_decode(const pa_bf16* q, const pa_bf16* k_cache, const pa_bf16* v_cache,
              const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
              int32_t max_context_len, float scale, pa_bf16* out, void* workspace,
              size_t workspace_bytes, const pa_cache_desc* desc, void* stream);
PA_API int pa_decode_ex(const pa_bf16* q, const pa_bf16* k_cache, const pa_bf16* v_cache,
                 const int32_t* block_tables, const int32_t* context_lens, int32_t num_seqs,
                 int32_t max_context_len, float scale, pa_bf16* out, void* workspace,
                 size_t workspace_bytes, const pa_cache_desc* desc,
                 const pa_decode_options* options, void* stream);

/*
 * One decode step in one call: for every sequence b with L = context_lens[b] > 0,
 * writes k[b], v[b] ([num_seqs][Hkv][D] bf16, all kv heads) into position L-1 of
 * its table row (slot = block_tables[b][(L-1)/Bs]*Bs + (L-1)%Bs), then runs
 * pa_decode over the L tokens.  The same result as pa_slot_mapping +
 * pa_append_kv + pa_decode; the tensor-core kernel writes the new rows itself,
 * just before it loads the block that holds them, which saves a launch and a
 * pass.  Same arguments and errors as pa_decode_ex plus k and v (16-byte
 * aligned); k_cache and v_cache are written.
 *
 * With options->rope_theta > 0, q[b] and k[b] are first turned by RoPE at
 * position L-1 (as pa_rope_append_kv does) and the rotated rows are rounded to
 * bf16: the cache receives the rotated K, and the rotated q attends.  q itself
 * is not modified.  The whole-group tensor kernel rotates in place of the
 * append; the other kernels run one rotation kernel first, which writes the
 * rotated q into the workspace (pa_decode_workspace_size_ex counts it when
 * given the same options).
 */
PA_API int pa_append_decode(const pa_bf16* q, const pa_bf16* k, const pa_bf16* v,
                            pa_bf16* k_cache, pa_bf16* v_cache, const int32_t* block_tables,
                            const int32_t* context_lens, int32_t num_seqs, int32_t max_context_len,
                            float scale, pa_bf16* out, void* workspace, size_t workspace_bytes,
                            const pa_cache_desc* desc, const pa_decode_options* options,
                            void* stream);

/*
 * Paged (chunked) prefill attention.  Prefill processes a prompt, or a chunk of
 * it, at once (Nano-vLLM page, "Nano-vLLM로 배우는 vLLM 추론 엔진 작동 원리 한눈에
 * 정리", section "Prefill vs Decode"); the causal mask lets a token see only
 * itself and earlier tokens (Tiny-vLLM summary page, section "고성능 추론을 위한
 * 고급 최적화 기법").  Sequence b holds L = context_lens[b] tokens in the paged
 * cache, this chunk's K/V included (append them first, e.g. pa_append_kv with
 * their slots); its Tq = cu_seqlens_q[b+1] - cu_seqlens_q[b] query rows of q
 * ([total_q][Hq][D] bf16, rows cu_seqlens_q[b] ..) sit at positions L-Tq .. L-1,
 * and the query at position p attends to cache tokens 0..p:
 *   out[row][h] = bf16( sum_{j<=p} softmax_j(scale * q[row][h] . K_j) V_j ),
 * K_j, V_j of kv head h / (Hq/Hkv).  fp32 accumulation, online softmax.
 * cu_seqlens_q: [num_seqs + 1] int32 device array (0 first, non-decreasing);
 * max_q_len >= every Tq (sizes the grid).  workspace: >= 256 bytes, 256-byte
 * aligned, its status word as for pa_decode (a block id outside the pool, or
 * L < Tq, L past the table or Tq > max_q_len: the sequence's rows are left
 * unwritten and pa_decode_status reports it).  head_dim 64 or 128.
 * kernel: PA_PREFILL_AUTO (PA_PREFILL_TCGEN05_WS where it serves the block
 * size, else PA_PREFILL_TCGEN05), PA_PREFILL_TCGEN05 (128-row tiles on the
 * fifth-generation tensor cores, accumulators in tensor memory),
 * PA_PREFILL_TCGEN05_WS (the same tiles with one job per warp) or
 * PA_PREFILL_MMA (64-row tiles on warp-level mma.sync); all compute the same
 * operation, with fp32 accumulation in a different order.
 * Errors: PA_ERR_INVALID (also an unknown kernel), PA_ERR_UNSUPPORTED,
 * PA_ERR_WORKSPACE, PA_ERR_CUDA.
 */
#define PA_PREFILL_AUTO     0
#define PA_PREFILL_TCGEN05  1
#define PA_PREFILL_MMA      2
#define PA_PREFILL_TCGEN05_WS 3   /* tcgen05 with one job per warp (softmax, MMA issue, TMA) and */
                                  /* O accumulated in tensor memory; block sizes 8, 16, 32, 64  */
                                  /* or multiples of 64 (PA_ERR_UNSUPPORTED otherwise)          */
PA_API int pa_prefill(const pa_bf16* q, const pa_bf16* k_cache, const pa_bf16* v_cache,
                      const int32_t* block_tables, const int32_t* cu_seqlens_q,
                      const int32_t* context_lens, int32_t num_seqs, int32_t max_q_len, float scale,
                      pa_bf16* out, void* workspace, size_t workspace_bytes,
                      const pa_cache_desc* desc, int32_t kernel, void* stream);

/*
 * Synchronises `stream`, reads and clears the workspace's device status word.
 * Returns PA_OK, PA_ERR_BAD_BLOCK, PA_ERR_BAD_LENGTH, PA_ERR_TIMEOUT or
 * PA_ERR_UNSUPPORTED (a tensor-core kernel found its shared memory off the
 * 1024-byte boundary its swizzled tiles need, and wrote nothing) -- the first
 * set, in that order -- or PA_ERR_CUDA if the read fails.
 */
PA_API int pa_decode_status(void* workspace, size_t workspace_bytes, void* stream);

/* Number of KV splits pa_decode uses per (sequence, kv head) at most for this shape. */
PA_API int32_t pa_decode_max_splits(int32_t num_seqs, int32_t max_context_len, const pa_cache_desc* desc,
                             const pa_decode_options* options);

/*
 * How pa_decode (and pa_append_decode, pa_decode_noalloc) will partition the work of a call
 * of this shape on the current device, for callers that size, test or profile around it.
 *  kernel:       PA_KERNEL_TENSOR for the stream-partitioned whole-group kernel (Hkv a
 *                multiple of 8), PA_KERNEL_TENSOR_SPLIT or PA_KERNEL_SIMT for the split ones.
 *  ctas:         stream kernel: CTAs of its persistent grid.  The work is the concatenation,
 *                over groups of 8 kv heads and then sequences, of slabs of split_tokens
 *                tokens (an empty sequence counts one); CTA i of G = min(ctas, slabs S) takes
 *                slabs [i S / G, (i + 1) S / G).  0 for the split kernels.
 *  split_tokens: split kernels: tokens per split (split k covers [k C, (k + 1) C)); stream
 *                kernel: tokens per slab (32 for E4M3 pools with head_dim 64, else 16).
 *  max_splits:   split kernels: splits per (sequence, kv head) at most; else 1.
 * Returns PA_OK, or the error the decode call itself would return for these arguments.
 */
typedef struct pa_decode_plan_info {
    int32_t kernel;
    int32_t ctas;
    int32_t split_tokens;
    int32_t max_splits;
} pa_decode_plan_info;

PA_API int pa_decode_describe(int32_t num_seqs, int32_t max_context_len, const pa_cache_desc* desc,
                              const pa_decode_options* options, pa_decode_plan_info* out);

/* ---- paged decode without allocation ------------------------------------------------------ */
/*
 * (The pages have no counterpart: this is a deployment convenience.)
 *
 * pa_decode for callers that cannot allocate device memory: code that runs
 * under a memory planner which owns every device allocation in advance (an
 * inference runtime that gives a plugin only its inputs and outputs), code on
 * a latency-bound path where a cudaMalloc could synchronise the device or fail
 * at the wrong moment, or C callers without an allocator.  Same arguments,
 * result and errors as pa_decode_ex, minus the workspace: the scratch comes
 * from a fixed array of PA_NOALLOC_SCRATCH_BYTES in the library's device image,
 * which every GPU that loads the library holds until the process exits.  The
 * call allocates nothing.
 *  - A shape whose workspace (pa_decode_workspace_size_ex) exceeds
 *    PA_NOALLOC_SCRATCH_BYTES returns PA_ERR_WORKSPACE and launches nothing.
 *  - The first call on each device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture.
 *  - Every call shares the one array and it keeps the previous call's
 *    contents (the words that must start at zero are cleared on `stream`), so
 *    calls that may overlap on the GPU race: serialise them (one stream).
 *  - Device-side errors (a block id outside the pool, a clipped length, a
 *    timed-out wait) are reported only with PA_FLAG_CHECK, which synchronises
 *    `stream` and returns them; without it they are dropped, because the next
 *    call clears the array's status word before it runs.
 *  - The clearing is a memset on `stream` between the previous kernel and the
 *    decode, so PA_FLAG_PDL gives no early start here.
 *  - The cached address is that of the device's primary context (the one the
 *    CUDA runtime uses); do not call this from another driver-API context on the
 *    same device.
 */
#define PA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

PA_API int pa_decode_noalloc(const pa_bf16* q, const pa_bf16* k_cache, const pa_bf16* v_cache,
                             const int32_t* block_tables, const int32_t* context_lens,
                             int32_t num_seqs, int32_t max_context_len, float scale, pa_bf16* out,
                             const pa_cache_desc* desc, const pa_decode_options* options,
                             void* stream);

/* ---- host slot mapping ----------------------------------------------------------------- */
/*
 * slots[b] = block_tables[b][p / Bs] * Bs + p % Bs with p = lengths[b] - 1
 * (the newest token's slot), or -1 when lengths[b] <= 0.  Host memory only.
 */
PA_API int pa_slot_mapping(const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* lengths, int32_t num_seqs, int32_t block_size, int64_t* slots);

/* ---- host block pool --------------------------------------------------------------------- */
/*
 * The allocator of the paged pool on its own (host memory): the KV cache is divided into
 * fixed-size blocks handed out only as tokens need them, and one block may sit in several
 * block tables at once (vLLM overview page, "vLLM — PagedAttention으로 LLM 추론 성능을 2~4배
 * 끌어올린 서빙 엔진" (dev.to), section "PagedAttention — OS 가상 메모리에서 영감"; Nano-vLLM
 * page, section "KV 캐시와 Block Manager", shared prefix blocks).  For callers that keep
 * their own block tables; pa_bm_* below applies the same policy and keeps the tables too.
 * Policy: free ids form a stack with free_order[0] on top; pa_pool_alloc takes n ids from the
 * top (all or nothing: PA_ERR_OOM_BLOCKS and no change when fewer are free) and gives each a
 * reference count of 1; pa_pool_share adds one holder to an allocated block; pa_pool_free
 * drops one, and at zero the block goes back on top of the stack.  Blocks not listed in
 * free_order start allocated with a count of 1.  Sharing or freeing a free block, or an id
 * outside [0, num_blocks), is PA_ERR_INVALID and changes nothing.  Not thread-safe.
 */
typedef struct pa_block_pool pa_block_pool;

PA_API int pa_pool_create(int32_t num_blocks, const int32_t* free_order, int32_t num_free,
                          pa_block_pool** out);
PA_API void pa_pool_destroy(pa_block_pool* pool);
/* n free blocks, top of the stack first, into blocks[0..n). */
PA_API int pa_pool_alloc(pa_block_pool* pool, int32_t n, int32_t* blocks);
PA_API int pa_pool_share(pa_block_pool* pool, int32_t block);
PA_API int pa_pool_free(pa_block_pool* pool, int32_t block);
PA_API int32_t pa_pool_num_free(const pa_block_pool* pool);
/* Holders of a block (0 = free), or -1 for an id outside the pool. */
PA_API int32_t pa_pool_refcount(const pa_block_pool* pool, int32_t block);

/* ---- host block manager ---------------------------------------------------------------- */
/*
 * Host-memory bookkeeping of a block pool shared by up to max_seqs sequence
 * rows.  Policy: free blocks form a stack, free_order[0] handed out first; a
 * block's reference count is the number of tables holding it and it returns
 * to the top of the stack when the count reaches zero; releasing a sequence
 * walks its table from logical block 0; appending a token at position p takes
 * a block when p % Bs == 0; a batch append is all-or-nothing; an append into
 * a block held by more than one table is refused (PA_ERR_SHARED_BLOCK).
 * Not thread-safe: one manager per thread.
 */
typedef struct pa_block_manager pa_block_manager;

PA_API int pa_bm_create(int32_t num_blocks, int32_t block_size, int32_t max_seqs,
                 int32_t max_blocks_per_seq, const int32_t* free_order, int32_t num_free,
                 pa_block_manager** out);
PA_API void pa_bm_destroy(pa_block_manager* bm);
/* Adopt a sequence whose num_tokens tokens already sit in `blocks` (ceil(num_tokens/Bs)
 * ids that are not on the free stack); each block's count rises by one. */
PA_API int pa_bm_import_seq(pa_block_manager* bm, int32_t seq, int32_t num_tokens, const int32_t* blocks);
/* Admit a sequence of num_tokens cached tokens into fresh blocks. */
PA_API int pa_bm_add_seq(pa_block_manager* bm, int32_t seq, int32_t num_tokens);
/* Admit a sequence that shares the first num_shared_blocks blocks of src (which must be
 * full) and gets fresh blocks for the rest of its num_tokens tokens. */
PA_API int pa_bm_fork_seq(pa_block_manager* bm, int32_t seq, int32_t src, int32_t num_shared_blocks,
                   int32_t num_tokens);
/* Release a sequence's blocks. */
PA_API int pa_bm_free_seq(pa_block_manager* bm, int32_t seq);
/* One new token for each of the n (distinct) listed sequences; slots[i] receives its slot. */
PA_API int pa_bm_append_tokens(pa_block_manager* bm, const int32_t* seqs, int32_t n, int64_t* slots);
PA_API int32_t pa_bm_num_free(const pa_block_manager* bm);
PA_API int32_t pa_bm_refcount(const pa_block_manager* bm, int32_t block);
/* Host views, valid until the manager is destroyed: [max_seqs][max_blocks_per_seq] (-1
 * past each sequence's blocks) and [max_seqs] (0 for rows without a sequence). */
PA_API const int32_t* pa_bm_block_tables(const pa_block_manager* bm);
PA_API const int32_t* pa_bm_context_lens(const pa_block_manager* bm);
/* Rows whose table changed since the last call (up to cap, ascending); returns the count. */
PA_API int32_t pa_bm_take_dirty_rows(pa_block_manager* bm, int32_t* rows, int32_t cap);

/*
 * ---- prefix caching and copy-on-write ----
 * The Nano-vLLM page ("Nano-vLLM로 배우는 vLLM 추론 엔진 작동 원리 한눈에 정리",
 * section "KV 캐시와 Block Manager") reuses the blocks of a shared prompt
 * prefix, identified by a hash, without recomputing them.  Here a FULL block
 * is identified by the 64-bit FNV-1a hash of its parent block's hash (8 bytes,
 * little-endian; 0 for the first block) followed by its Bs token ids (4 bytes
 * each, little-endian); a lookup hits only when the stored ids are equal too.
 * Copy-on-write follows the OS paging the vLLM overview page likens the pool
 * to (section "PagedAttention — OS 가상 메모리에서 영감"): an append into a
 * block that several tables hold first moves the writer to a fresh block.
 * Free-list policy: a block freed without a hash returns to the top (the
 * stack above, unchanged); a freed hashed block stays cached at the bottom
 * (a sequence's blocks tail first, so a prefix outlives its extensions) until
 * allocation reaches it, which evicts its hash.  A sequence's blocks are
 * hashed while every token it holds has an id (admitted by
 * pa_bm_add_seq_tokens, grown by pa_bm_append_token_ids, or forked whole from
 * such a sequence); a block is registered when it fills, unless its hash is
 * already registered.  The caller fills the KV of the blocks that were not
 * found cached (prefill) and runs the reported copies (pa_copy_blocks) before
 * the appends that follow them.
 */
/* Admit a sequence by its num_tokens token ids; the blocks of its longest cached prefix of
 * full blocks are shared, the rest are fresh.  *num_cached_tokens (may be NULL) receives the
 * number of tokens found cached (a multiple of Bs).  All-or-nothing: PA_ERR_OOM_BLOCKS when the
 * free list cannot cover the fresh blocks (cached free blocks that hit do not count as fresh). */
PA_API int pa_bm_add_seq_tokens(pa_block_manager* bm, int32_t seq, const int32_t* token_ids,
                                int32_t num_tokens, int32_t* num_cached_tokens);
/* Admit seq as a copy of src sharing every block, its partial last block included (for
 * parallel sampling); the first append of either into the shared partial block copies it. */
PA_API int pa_bm_fork_all(pa_block_manager* bm, int32_t seq, int32_t src);
/* pa_bm_append_tokens with token ids and copy-on-write: token token_ids[i] is appended to
 * seqs[i] (n distinct sequences) and slots[i] receives its slot.  When the token lands in a
 * block other tables also hold, the sequence gets a fresh block first and the pair (old,
 * fresh) is written to copies[2 k], copies[2 k + 1] (capacity 2 n), k < *num_copies.
 * All-or-nothing on PA_ERR_OOM_BLOCKS. */
PA_API int pa_bm_append_token_ids(pa_block_manager* bm, const int32_t* seqs, const int32_t* token_ids,
                                  int32_t n, int64_t* slots, int32_t* copies, int32_t* num_copies);
/* Number of registered (hash-identified) blocks, in use or cached free. */
PA_API int32_t pa_bm_num_cached_blocks(const pa_block_manager* bm);

/*
 * Device side of copy-on-write: for k < n, block copies[2 k + 1] of k_cache and of v_cache
 * receives a bit-exact copy of block copies[2 k] (all kv heads, all Bs slots).  copies is a
 * device int32 array [n][2]; ids outside [0, num_blocks) skip that pair; destinations must
 * be distinct and no destination may be a source of another pair.  Caches 16-byte aligned,
 * head_dim a multiple of 8.  n == 0 is a no-op.  Errors: PA_ERR_INVALID, PA_ERR_CUDA.
 */
PA_API int pa_copy_blocks(pa_bf16* k_cache, pa_bf16* v_cache, const int32_t* copies, int32_t n,
                          const pa_cache_desc* desc, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
