/*
 * fa.h — C ABI of the B200 (sm_100a) exact-attention library libfa.so.
 *
 * What it computes (sources are web pages on FlashAttention/PagedAttention):
 *   O = softmax(scale * Q K^T [+ causal mask]) V, one pass over K/V tiles with
 *   a running row max m and running row sum l, the unnormalised output
 *   rescaled by exp(m_old - m_new) and divided by l once at the end, plus the
 *   per-row logsumexp L = m + log l
 *     - "FlashAttention系列优化" (johneyzheng.top), sections FlashAttentionV1
 *       (online softmax) and FlashAttentionV2 (delayed rescaling, Q-outer /
 *       KV-inner loop order);
 *     - FlashAttention v1/v2/v3 overview (91haoming.cn repost), "前向傳播改進"
 *       (store only L = m + log l) and "并行化改進" (parallel over row blocks
 *       forward, over column blocks backward);
 *     - "Flash Attention 再学习" (jibinghu.github.io): 1-pass tiling, backward
 *       by recomputing S and P from the stored statistics.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers, owned by the caller, at least
 *     16-byte aligned (TMA requirement); the library keeps no reference to them
 *     after the call returns.
 *   - "BHND" = [B][H][N][d] contiguous row-major; bf16 = IEEE bfloat16 bits.
 *   - Softmax scale is fixed at 1/sqrt(d). Scores, L and all accumulation are
 *     fp32. L is the natural-log logsumexp of the scaled scores.
 *   - Causal: query row i attends key j iff j <= i (same N for Q and K).
 *   - d must be 64 or 128 (FA_ERR_UNSUPPORTED otherwise); N >= 1; any N is
 *     allowed (ragged last tiles are masked / zero-filled).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). A non-FA_OK return means nothing was launched.
 *   - Every wait inside a kernel is bounded; a wait that gives up records an
 *     error in a device-side word and the kernel returns early. Such failures
 *     surface through fa_last_device_error(), not through the launch status.
 *   - The library holds no global state apart from a per-device cache of
 *     device attributes and the device error word.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

/* Symbols the shared library exports (it is built with hidden visibility). */
#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,  /* null / misaligned pointer, non-positive size */
  FA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d not 64/128) */
  FA_ERR_LAUNCH = 3,       /* CUDA runtime refused the launch */
  FA_ERR_TIMEOUT = 4,      /* a bounded in-kernel wait gave up */
  FA_ERR_WORKSPACE = 5     /* workspace missing or too small */
} fa_status;

/* Human-readable name of a status code (static string, never NULL). */
FA_API const char* fa_status_str(fa_status s);

/*
 * fa_fwd — fused one-pass attention forward.
 *   q, k, v : bf16 BHND inputs.
 *   o       : bf16 BHND output, O = diag(l)^-1 * sum_j exp(S_j - m) V_j
 *             rounded to bf16 (round to nearest even).
 *   lse     : fp32 [B][H][N] output, L = m + log(l) (natural log), the only
 *             softmax statistic kept for the backward.
 * Partitioning: one CTA per (batch, head, pair of 128-row Q tiles); K/V tiles
 * of 128 rows stream through a shared-memory ring ("并行化改進": row blocks are
 * independent, no communication between CTAs).
 * Errors: FA_ERR_INVALID_ARG for null/misaligned pointers or B, H, N < 1;
 * FA_ERR_UNSUPPORTED for d not in {64, 128}; FA_ERR_LAUNCH if CUDA fails.
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, int causal, void* stream);

/*
 * Bytes of device workspace fa_bwd needs: two fp32 per-row vectors over N
 * rounded up to a multiple of 128 rows — the row statistic D and L * log2(e)
 * (padded with 0 / +inf) — a small block of per-tensor statistics (the
 * largest magnitudes of q, k, v, dout and the power-of-two exponents chosen
 * from them), plus room for fp16 copies of q, k, v and dout (the backward's
 * tensor-core operands: fa_bwd and fa_bwd_dropout write the copies of q and
 * dout and convert k and v inside the main pass; fa_bwd_fp8 writes all
 * four), each part rounded up to 256 bytes. dq itself (fp32) serves as the dQ
 * accumulator.
 */
FA_API size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * fa_bwd — attention backward by recomputation.
 *   q, k, v, o, dout : bf16 BHND (o = fa_fwd's output, dout = dL/dO).
 *   lse              : fp32 [B][H][N] from fa_fwd.
 *   dq, dk, dv       : fp32 BHND outputs (gradients w.r.t. q, k, v).
 *   workspace        : device buffer of >= fa_bwd_workspace_bytes() bytes,
 *                      owned by the caller; contents on entry are ignored.
 * Steps: D_i = sum_c dO_ic O_ic (and dq := 0); then, per K/V column block j
 * (one CTA),
 * P = exp(scale*Q_i K_j^T - L_i) for every Q row block i it sees,
 * dV_j += P^T dO_i, dP = dO_i V_j^T, dS = P o (dP - D_i),
 * dK_j += scale dS^T Q_i, and dQ_i += scale dS K_j accumulated across CTAs
 * with fp32 reductions; dK_j and dV_j are written once.
 * ("Flash Attention 再学习": backward recomputes S and P from the stored
 * statistics; 91haoming.cn repost, "并行化改進": backward is parallel over
 * column blocks with atomic adds for the shared gradient.)
 * Precision: the products run on fp16 tensor-core operands with fp32
 * accumulation. Each of q, k, v, dout is first multiplied by a power of two
 * chosen from its largest magnitude a (so that it fits fp16's range); that
 * scaling is exact, and the fp16 copy of an element x is exact whenever
 * |x| >= 2^-30 a (smaller ones are off by less than 2^-38 a), so every
 * finite bf16 input is accepted and results do not depend on the inputs'
 * binade. The factors are undone in fp32. P and dS are rounded to fp16 (3
 * more mantissa bits than bf16), dS after a power-of-two scale that keeps it
 * below 2^15 when L is fa_fwd's L; a dS beyond fp16's range (an inconsistent
 * L) is reported by fa_last_device_error() as FA_ERR_UNSUPPORTED. Inputs so
 * large that scale * |q| * |k| leaves fp32's range give non-finite results,
 * as in the forward.
 * Errors: as fa_fwd, plus FA_ERR_WORKSPACE when workspace is NULL or smaller
 * than required.
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o,
                 const float* lse, const void* dout, float* dq, float* dk, float* dv,
                 void* workspace, size_t ws_bytes,
                 int B, int H, int N, int d, int causal, void* stream);

/*
 * fa_fwd_varlen — the forward over a packed batch of variable-length
 * sequences, with query and key lengths that may differ and grouped KV heads.
 * Same method as fa_fwd; the layouts generalise its BHND view: every (sequence,
 * head) is an independent problem ("Flash Attention 再学习", Flash Attention
 * v2, thread blocks parallel over batch, heads and row blocks).
 *   q, o          : bf16 [total_q][H][d], token-major; sequence b owns rows
 *                   [cu_seqlens_q[b], cu_seqlens_q[b+1]).
 *   k, v          : bf16 [total_k][Hkv][d]; sequence b owns rows
 *                   [cu_seqlens_k[b], cu_seqlens_k[b+1]).
 *   lse           : fp32 [H][total_q], natural log.
 *   cu_seqlens_q/k: int32 [batch + 1] device arrays, non-decreasing,
 *                   cu[0] = 0, cu[batch] <= total. Every query length must be
 *                   <= max_seqlen_q (it sizes the grid); key lengths may be 0.
 *   H, Hkv        : query head h reads KV head h / (H / Hkv); H % Hkv == 0.
 *   causal        : aligned to the bottom right, so query i of a sequence with
 *                   Lq queries and Lk keys sees keys j <= i + Lk - Lq (for
 *                   Lq == Lk this is fa_fwd's mask; for Lq = 1 the query sees
 *                   every key, as in decoding). A query that sees no key
 *                   (Lq > Lk, or Lk = 0) gets O = 0 and L = -inf.
 * The inputs must be finite (rows of the next sequence are read and masked).
 * Errors: FA_ERR_INVALID_ARG for NULL / unaligned pointers, batch, H, Hkv,
 * max_seqlen_q, totals < 1, H % Hkv != 0 or max_seqlen_q > total_q;
 * FA_ERR_UNSUPPORTED for d not in {64, 128} or sizes beyond 32-bit indexing;
 * FA_ERR_LAUNCH as fa_fwd. Inconsistent cu_seqlens (a length < 0, a query
 * length > max_seqlen_q, or a range past the totals) are detected on the
 * device: that sequence is skipped and fa_last_device_error() reports
 * FA_ERR_INVALID_ARG.
 */
FA_API fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int batch,
                        int max_seqlen_q, int total_q, int total_k, int H, int Hkv, int d,
                        int causal, void* stream);

/*
 * fa_bwd_varlen_workspace_bytes — device workspace fa_bwd_varlen needs: D and
 * L log2(e) for [batch][H][max_seqlen_q rounded up to 128] rows, and room for
 * fp16 copies of q, k, v, dout (those of q and dout are written; k and v are
 * converted inside the main pass). 0 for invalid sizes.
 */
FA_API size_t fa_bwd_varlen_workspace_bytes(int batch, int max_seqlen_q, int total_q,
                                            int total_k, int H, int Hkv, int d);

/*
 * fa_bwd_varlen — gradients of fa_fwd_varlen (same method as fa_bwd: P rebuilt
 * from L, dQ accumulated across key blocks; layouts and the bottom-right causal
 * mask as fa_fwd_varlen).
 *   q, o, dout    : bf16 [total_q][H][d]; lse fp32 [H][total_q] from fa_fwd_varlen.
 *   k, v          : bf16 [total_k][Hkv][d].
 *   dq            : fp32 [total_q][H][d]; rows of the sequences are written
 *                   (rows past cu_seqlens_q[batch] are left as they are).
 *   dk, dv        : fp32 [total_k][Hkv][d]; a KV head's gradient sums its
 *                   group's query heads; rows past cu_seqlens_k[batch] untouched.
 *   max_seqlen_q/k: bounds on every query / key length (they size the grid).
 *   d             : 128 only for now (FA_ERR_UNSUPPORTED otherwise).
 * Precision as fa_bwd (fp16 operands, |x| < 65504). Errors as fa_fwd_varlen,
 * plus FA_ERR_WORKSPACE when the workspace is NULL or smaller than
 * fa_bwd_varlen_workspace_bytes().
 */
FA_API fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, float* dq, float* dk, float* dv,
                        void* workspace, size_t ws_bytes, const int* cu_seqlens_q,
                        const int* cu_seqlens_k, int batch, int max_seqlen_q, int max_seqlen_k,
                        int total_q, int total_k, int H, int Hkv, int d, int causal,
                        void* stream);

/*
 * fa_paged_prefill — a chunk of new tokens per sequence attending to that
 * sequence's paged KV cache ("FlashAttention系列优化", PagedAttention: the
 * keys are reached through the block table, as in paged_attn_decode; the
 * chunk is a prefill or an append of several tokens at once).
 *   q, o          : bf16 [total_q][Hq][d]; sequence s's chunk is rows
 *                   [cu_seqlens_q[s], cu_seqlens_q[s+1]); lse fp32 [Hq][total_q].
 *   k_cache, v_cache, num_phys_blocks, block_table, max_blocks_per_seq:
 *                   as paged_attn_decode ([P][Hkv][16][d] bf16; int32 table
 *                   [batch][max_blocks_per_seq]).
 *   context_lens  : int32 [batch], the cached tokens of each sequence,
 *                   including the chunk's own (already written), so the chunk
 *                   is the last Lq of its context_lens[s] tokens.
 *   causal        : bottom-right, as fa_fwd_varlen: chunk query i sees cached
 *                   tokens j <= context_lens[s] - Lq + i (0: every cached token).
 *   d in {64, 128}, block_size 16, Hq % Hkv == 0.
 * Errors as fa_fwd_varlen; a table entry outside [0, num_phys_blocks) is never
 * dereferenced (block 0 is read instead) and is reported, like a context
 * longer than max_blocks_per_seq * 16, by fa_last_device_error() as
 * FA_ERR_INVALID_ARG.
 */
FA_API fa_status fa_paged_prefill(const void* q, const void* k_cache, const void* v_cache,
                           int num_phys_blocks, const int* block_table, int max_blocks_per_seq,
                           const int* cu_seqlens_q, const int* context_lens, void* o, float* lse,
                           int batch, int max_seqlen_q, int total_q, int Hq, int Hkv, int d,
                           int block_size, int causal, void* stream);

/*
 * fa_fwd_block_sparse — fa_fwd restricted to the (query block, key block)
 * pairs a block mask keeps, blocks of 128 x 128 ("91haoming.cn" repost,
 * FlashAttention v1, 實現效果: block-sparse FlashAttention; skipped blocks are
 * neither loaded nor computed unless the other query tile of the CTA needs
 * them, in which case they are masked).
 *   block_mask     : uint8 device array; query block qb sees key block kb iff
 *                    block_mask[bh * mask_bh_stride + qb * nb + kb] != 0, with
 *                    nb = ceil(N / 128) and bh = b * H + h; mask_bh_stride = 0
 *                    shares one nb x nb mask across all (b, h), otherwise it
 *                    must be >= nb * nb.
 *   causal         : applied on top of the block mask (key j <= query i).
 *   A query that sees no key gets O = 0 and L = -inf. N <= 65536.
 * Other arguments, layouts and errors as fa_fwd.
 */
FA_API fa_status fa_fwd_block_sparse(const void* q, const void* k, const void* v, void* o,
                              float* lse, const unsigned char* block_mask,
                              long long mask_bh_stride, int B, int H, int N, int d, int causal,
                              void* stream);

/*
 * fa_fwd_dropout — fa_fwd with dropout on the attention probabilities
 * ("91haoming.cn" repost, FlashAttention v1, 注意力實現改進: the matmuls, the
 * softmax, the optional mask and dropout run in one fused kernel; the pages
 * give no formula, so the contract is fixed here):
 *   O = (P o Z) V / q_keep,  P = softmax(S / sqrt(d) [+ causal mask]);
 *   lse is that of the undropped scores, exactly as fa_fwd writes it.
 *   Z (keep mask): element (b, h, i, j) (query i, key j) is kept iff
 *     byte (j % 16) of Philox4x32-10(counter = (j / 16, i, b * H + h, offset),
 *     key = (seed & 0xffffffff, seed >> 32)) >= t, bytes numbered from the
 *     low byte of output word 0 to the high byte of word 3 (Philox4x32-10:
 *     Salmon et al., "Parallel random numbers: as easy as 1, 2, 3", SC 2011).
 *   t = floor(256 * p_drop + 0.5) is the drop threshold; q_keep = 1 - t / 256.
 *   p_drop: 0 <= p_drop and t <= 255, else FA_ERR_INVALID_ARG. The applied drop
 *   probability is t / 256 (a multiple of 1/256).
 * The same (seed, offset) in fa_bwd_dropout regenerates the same Z. Other
 * arguments, layouts and errors as fa_fwd.
 */
FA_API fa_status fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int N, int d, int causal, float p_drop,
                                unsigned long long seed, unsigned int offset, void* stream);

/*
 * fa_bwd_dropout — gradients of fa_fwd_dropout with its keep mask Z:
 *   dV = (P o Z)^T dO / q_keep,  dP = Z o (dO V^T) / q_keep,
 *   D_i = sum_c dO_ic O_ic (o = the dropout forward's output),
 *   dS = P o (dP - D),  dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d).
 *   p_drop, seed, offset: those given to fa_fwd_dropout.
 *   d = 64 or 128 (FA_ERR_UNSUPPORTED otherwise).
 * Workspace (fa_bwd_workspace_bytes), precision, other arguments and errors
 * as fa_bwd.
 */
FA_API fa_status fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, float* dq, float* dk,
                                float* dv, void* workspace, size_t ws_bytes, int B, int H, int N,
                                int d, int causal, float p_drop, unsigned long long seed,
                                unsigned int offset, void* stream);

/*
 * Bytes of device workspace paged_attn_decode needs for split partials
 * (fp32 O and L per (sequence, query head, split)) and a work counter, when
 * no sequence is longer than max_ctx tokens.
 */
FA_API size_t paged_attn_decode_workspace_bytes(int num_seqs, int Hq, int d, int max_ctx);

/*
 * paged_attn_decode — one query token per sequence against a paged KV cache.
 *   q            : bf16 [num_seqs][Hq][d].
 *   k_cache,
 *   v_cache      : bf16 [num_phys_blocks][Hkv][block_size][d]; one
 *                  (block, kv head) is block_size*d contiguous elements.
 *   num_phys_blocks : number of physical blocks in each cache; a table entry
 *                  outside [0, num_phys_blocks) is never dereferenced: the
 *                  kernel reads block 0 in its place and records the error,
 *                  which fa_last_device_error() reports as FA_ERR_INVALID_ARG.
 *   block_table  : int32 [num_seqs][max_blocks_per_seq]; token t of sequence s
 *                  is in physical block block_table[s][t / block_size] at slot
 *                  t % block_size ("FlashAttention系列优化", PagedAttention:
 *                  logical blocks map to physical blocks through a table;
 *                  several sequences may map to the same physical block).
 *                  Entries past ceil(ctx/block_size) are never read.
 *   context_lens : int32 [num_seqs], each in [1, max_ctx]; a length outside
 *                  that range is reported by fa_last_device_error() as
 *                  FA_ERR_INVALID_ARG (the kernels then use it clamped into
 *                  the range, so nothing outside the table or the workspace is
 *                  read or written, and that sequence's output is undefined).
 *   o            : bf16 [num_seqs][Hq][d] output.
 *   lse          : fp32 [num_seqs][Hq] output, or NULL to skip it.
 *   Query head h reads KV head h / (Hq / Hkv), with 1 <= Hq / Hkv <= 8 (one
 *   work item serves the query heads of one KV head, so each K/V byte is read
 *   once per group). d is 64 or 128. The query attends to all
 *   context_lens[s] cached tokens (no mask).
 *   workspace    : >= paged_attn_decode_workspace_bytes(num_seqs, Hq, d,
 *                  max_ctx) bytes; max_ctx must bound every context length.
 * Each (sequence, KV head, split of the context) is one CTA producing a
 * partial (O_s, L_s); a second kernel merges them:
 * L = log sum_s exp(L_s), O = sum_s exp(L_s - L) O_s.
 * Errors: FA_ERR_INVALID_ARG (null/misaligned pointers, sizes < 1, Hq not a
 * multiple of Hkv, a table narrower than max_ctx); FA_ERR_UNSUPPORTED (d not
 * 64 or 128, block_size != 16, Hq/Hkv > 8); FA_ERR_WORKSPACE; FA_ERR_LAUNCH.
 * Context lengths and table entries are read on the device and checked there
 * (see context_lens and num_phys_blocks).
 */
FA_API fa_status paged_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                            int num_phys_blocks, const int* block_table, int max_blocks_per_seq,
                            const int* context_lens, void* o, float* lse,
                            int num_seqs, int Hq, int Hkv, int d, int block_size,
                            int max_ctx, void* workspace, size_t ws_bytes, void* stream);

/*
 * paged_attn_decode_noalloc — paged_attn_decode without a workspace argument,
 * for callers that cannot allocate device memory on their decode path (for
 * example an engine that fixes its whole device-memory plan at start-up and
 * forbids allocation afterwards, or code that must not trigger the implicit
 * synchronisation of cudaMalloc/cudaFree). The pages have no counterpart: this
 * is an interface convenience around the same two kernels.
 * The split partials go to a 16 MiB device array inside the library (every
 * GPU that loads the library holds it until the process exits); the call
 * allocates nothing. Arguments, layouts and results are those of
 * paged_attn_decode.
 *   - Limit: paged_attn_decode_workspace_bytes(num_seqs, Hq, d, max_ctx) must
 *     not exceed 16 MiB (16777216 bytes); larger requests return
 *     FA_ERR_WORKSPACE and launch nothing.
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture.
 *   - All calls share the array and it keeps the last call's contents. Each
 *     call clears what must start at zero (its work counter) itself, and every
 *     partial it reads was written by the same call. Calls that overlap on
 *     the GPU (different streams, or several host threads) race on it and
 *     must be serialised by the caller.
 */
FA_API fa_status paged_attn_decode_noalloc(const void* q, const void* k_cache,
                                           const void* v_cache, int num_phys_blocks,
                                           const int* block_table, int max_blocks_per_seq,
                                           const int* context_lens, void* o, float* lse,
                                           int num_seqs, int Hq, int Hkv, int d, int block_size,
                                           int max_ctx, void* stream);

/*
 * fa_fp8_prepare — incoherent processing + per-block e4m3 quantisation.
 *   q, k, v    : bf16 BHND inputs.
 *   R          : fp32 [d][d] orthogonal matrix (row-major); Q' = Q R and
 *                K' = K R, so Q'K'^T = Q K^T ("FlashAttention系列优化",
 *                FlashAttentionV3: multiply Q and K by a random orthogonal
 *                matrix to spread outliers without changing the result).
 *   q8, k8, v8 : e4m3 BHND outputs (1 byte per element).
 *   sq, sk, sv : fp32 [B][H][ceil(N/64)] per-block scales: a block is 64 token
 *                rows x d of one (b, h); scale = amax / 448 (1 if the block is
 *                all zero), x8 = round_to_nearest_even(x / scale) saturated to
 *                +-448 ("block quantization": one scale per block).
 * Precision of the rotation: d = 128 runs Q R and K R on the tensor core
 * with the bf16 inputs exact and R split into two bf16 terms (R = hi + lo,
 * |R - hi - lo| <= 2^-18 |R|), accumulating in fp32, so each rotated value is
 * within (2^-18 + 2 d 2^-23) sum_c |x_c R_c| of the exact product; d = 64
 * rotates in fp32 on the CUDA cores. A value that lands that close to an e4m3
 * rounding boundary may take the neighbouring code.
 * Errors: as fa_fwd (d must be 64 or 128).
 */
FA_API fa_status fa_fp8_prepare(const void* q, const void* k, const void* v, const float* R,
                         void* q8, void* k8, void* v8, float* sq, float* sk, float* sv,
                         int B, int H, int N, int d, void* stream);

/*
 * fa_fwd_fp8 — attention forward on e4m3 inputs with per-block scales.
 *   q8, k8, v8 : e4m3 BHND (from fa_fp8_prepare); sq, sk, sv their scales.
 *   o          : bf16 BHND output; lse: fp32 [B][H][N].
 * S = scale * sq_i * sk_j * (q8 k8^T) per 64-row block pair; the V block
 * scale is folded into P before P is rounded to e4m3 for the P.V product.
 * Errors: as fa_fwd (d must be 64 or 128).
 */
FA_API fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8,
                     const float* sq, const float* sk, const float* sv,
                     void* o, float* lse, int B, int H, int N, int d, int causal,
                     void* stream);

/*
 * fa_bwd_fp8 — the backward of the FP8 forward ("FlashAttention系列优化",
 * FlashAttentionV3 / FP低精度; 91haoming.cn repost, "FP8 低精度計算"; the
 * pages give no FP8 backward). It returns the gradients with respect to the
 * forward's own inputs q, k, v (before rotation and quantisation), treating
 * the e4m3 block quantisation as the identity (straight through):
 *   (dQ', dK', dV) = attention backward over Q' = q8 * sq, K' = k8 * sk,
 *                    V = v8 * sv (the dequantised 64-row blocks), D from o,
 *   dQ = dQ' R^T,  dK = dK' R^T    (R orthogonal: Q' = Q R).
 *   q8, k8, v8, sq, sk, sv : exactly what fa_fp8_prepare returned (and
 *                    fa_fwd_fp8 consumed); R the rotation given to it.
 *   o, lse         : fa_fwd_fp8's outputs (bf16 BHND, fp32 [B][H][N]).
 *   dout           : bf16 BHND; dq, dk, dv fp32 BHND outputs.
 *   workspace      : >= fa_bwd_workspace_bytes(B, H, N, d) bytes.
 * The products run on fp16 tensor-core operands: the e4m3 codes are fp16
 * values exactly (so the recomputed scores are the forward's), dout is
 * scaled by a power of two as in fa_bwd, and every block scale is applied in
 * fp32. e4m3 gradient operands were not used: rounding dout to e4m3 alone
 * moves dV by ~1 on the FP8 workload (tolerance 5e-2). The rotation back is a
 * second pass over dq and dk.
 * Errors: as fa_bwd; FA_ERR_UNSUPPORTED unless d = 64 or 128.
 */
FA_API fa_status fa_bwd_fp8(const void* q8, const void* k8, const void* v8, const float* sq,
                            const float* sk, const float* sv, const float* R, const void* o,
                            const float* lse, const void* dout, float* dq, float* dk, float* dv,
                            void* workspace, size_t ws_bytes, int B, int H, int N, int d,
                            int causal, void* stream);

/*
 * Paged KV-cache block pool ("FlashAttention系列优化", PagedAttention: blocks
 * allocated on demand as tokens arrive; sequences of parallel sampling share
 * physical blocks through their block tables; a reference count per block and
 * copy-on-write keep sharing safe). Host-side, not thread-safe: the caller
 * serialises calls on one pool. Policy: the lowest-numbered free block is
 * handed out; an append to a sequence whose last block is partially filled and
 * shared first copies that block (copy-on-write), then takes new blocks in
 * order; every operation either completes or changes nothing.
 *
 * fa_kv_pool_create  — num_blocks physical blocks of block_size tokens, sequence
 *                      ids [0, max_seqs), at most max_blocks_per_seq blocks per
 *                      sequence. *out receives the pool (free with
 *                      fa_kv_pool_destroy). FA_ERR_INVALID_ARG for sizes < 1 or
 *                      out == NULL; FA_ERR_WORKSPACE if host memory runs out.
 * fa_kv_seq_add      — start an empty sequence (id must be unused).
 * fa_kv_seq_fork     — child (unused id) maps the parent's blocks and length;
 *                      each block gains a reference.
 * fa_kv_seq_free     — each of the sequence's blocks loses a reference (freed
 *                      at zero); the id becomes unused.
 * fa_kv_seq_append   — reserve slots for n_tokens after the last token. When a
 *                      copy-on-write happens, *n_copies = 1 and copy_src[0] /
 *                      copy_dst[0] name the blocks whose contents must be copied
 *                      on the device (fa_kv_copy_blocks) before the new tokens
 *                      are written; otherwise *n_copies = 0. Returns
 *                      FA_ERR_INVALID_ARG for an unused id, n_tokens < 0 or more
 *                      than max_blocks_per_seq blocks; FA_ERR_WORKSPACE when the
 *                      pool has too few free blocks (the pool is the workspace).
 * fa_kv_num_free / fa_kv_refcount / fa_kv_seq_len — queries (-1 for an invalid
 *                      pool, block or unused sequence).
 * fa_kv_block_table  — rows of the int32 table [n][max_blocks_per_seq] for the
 *                      given sequences (entries past ceil(len / block_size) are
 *                      0, which paged_attn_decode never reads) and their lengths.
 * fa_kv_copy_blocks  — on `stream`, copy block src[i] to block dst[i] in both
 *                      caches (device int32 arrays of n pairs; block_bytes = the
 *                      bytes of one physical block of one cache, a multiple of
 *                      16, e.g. Hkv * block_size * d * 2 for the
 *                      [P][Hkv][block_size][d] bf16 caches of paged_attn_decode).
 *                      Out-of-range block ids are skipped and reported by
 *                      fa_last_device_error() as FA_ERR_INVALID_ARG.
 */
typedef struct fa_kv_pool fa_kv_pool;
FA_API fa_status fa_kv_pool_create(int num_blocks, int block_size, int max_seqs,
                                   int max_blocks_per_seq, fa_kv_pool** out);
FA_API void fa_kv_pool_destroy(fa_kv_pool* pool);
FA_API fa_status fa_kv_seq_add(fa_kv_pool* pool, int seq);
FA_API fa_status fa_kv_seq_fork(fa_kv_pool* pool, int parent, int child);
FA_API fa_status fa_kv_seq_free(fa_kv_pool* pool, int seq);
FA_API fa_status fa_kv_seq_append(fa_kv_pool* pool, int seq, int n_tokens, int* copy_src,
                                  int* copy_dst, int* n_copies);
FA_API int fa_kv_num_free(const fa_kv_pool* pool);
FA_API int fa_kv_refcount(const fa_kv_pool* pool, int block);
FA_API int fa_kv_seq_len(const fa_kv_pool* pool, int seq);
FA_API fa_status fa_kv_block_table(const fa_kv_pool* pool, const int* seqs, int n, int* table,
                                   int max_blocks_per_seq, int* lens);
FA_API fa_status fa_kv_copy_blocks(void* k_cache, void* v_cache, int num_blocks, const int* src,
                                   const int* dst, int n, long long block_bytes, void* stream);

/*
 * fa_last_device_error — synchronises `stream`, then reads and clears the
 * device error word of the current device. Returns FA_OK when nothing was
 * recorded since the last call, FA_ERR_TIMEOUT when a bounded wait gave up,
 * FA_ERR_INVALID_ARG when a kernel met an out-of-range index in its inputs
 * (a block-table entry, a context length), FA_ERR_UNSUPPORTED when a value
 * left a kernel's numeric range (fa_bwd: a dS beyond fp16's range, which
 * only an L inconsistent with the scores produces), or FA_ERR_LAUNCH when the
 * synchronisation failed.
 * The word is one per device and process, shared by every stream and host
 * thread: the first error recorded by any kernel of the library on that
 * device is kept until some caller reads it here, and reading clears it for
 * all. Callers that run the library from several streams or threads at once
 * should read it at a point where they know which of their calls ran.
 */
FA_API fa_status fa_last_device_error(void* stream);

/*
 * fa_debug_wait_timeout — launches one CTA that waits on a shared-memory
 * barrier nothing ever arrives at, using the same bounded wait as the
 * kernels above, with a limit of `timeout_us` microseconds (1..1000000).
 * The wait gives up, records FA_ERR_TIMEOUT in the device error word and
 * the kernel returns. Exists so tests can check the failure path without
 * faulting or hanging a GPU.
 */
FA_API fa_status fa_debug_wait_timeout(unsigned int timeout_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
