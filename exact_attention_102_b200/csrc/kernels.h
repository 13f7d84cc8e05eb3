// kernels.h — launch interfaces between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

struct FwdArgs {
  void* o;            // bf16 [B][H][N][D]            (packed mode: [Tq][H][D])
  float* lse;         // fp32 [B][H][N]               (packed mode: [H][Tq])
  int B, H, N;        // packed mode: N = the longest query sequence
  int causal;
  int n_pairs;        // ceil(N / 256): pairs of 128-row Q tiles per head
  float scale_log2;   // softmax scale * log2(e)
  uint32_t* err;      // device error word
  // packed variable-length mode when cu_q != nullptr: sequence b owns query
  // rows [cu_q[b], cu_q[b+1]) of Q / O and key rows [cu_k[b], cu_k[b+1]) of
  // K / V; query head h reads KV head h / (H / Hkv); causal is aligned to the
  // bottom right (query i of Lq sees keys j <= i + Lk - Lq)
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int Hkv = 0, Tq = 0, Tk = 0;
  // paged K / V (packed mode with block_table != nullptr; cu_k unused): the
  // keys of sequence b are its ctx[b] cached tokens, token t in physical
  // block block_table[b * max_blocks + t / 16] at slot t % 16, i.e. row
  // (block * Hkv + kv head) * 16 + t % 16 of the [P * Hkv * 16][D] cache view
  const int* block_table = nullptr;
  const int* ctx = nullptr;
  int max_blocks = 0, num_phys = 0;
  // block-sparse [B, H, N, d] form (block_mask != nullptr): query block qb sees
  // key block kb iff block_mask[bh * mask_bh_stride + qb * ceil(N / 128) + kb]
  const uint8_t* block_mask = nullptr;
  long long mask_bh_stride = 0;
  // dropout on P ([B, H, N, d] form): element (b, h, i, j) is kept iff byte
  // j % 16 of Philox4x32-10((j / 16, i, b*H + h, drop_offset), (seed_lo,
  // seed_hi)) is >= t; drop_bias = (32768 - 128 t) * 0x00010001;
  // drop_scale = 256 / (256 - t) multiplies O
  int dropout = 0;
  uint32_t drop_bias = 0, seed_lo = 0, seed_hi = 0, drop_offset = 0;
  float drop_scale = 1.f;
  // [B, H, N, d] forms: (batch, head) slices per grid group (<= 0: one group
  // of all slices, i.e. heaviest pair first over every head)
  int head_group = 0;
};

template <int D>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdArgs& a, cudaStream_t stream);

struct BwdArgs {
  const void* q;      // bf16 BHND
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;   // fp32 [B][H][N]
  float* dq;          // fp32 BHND (accumulated with reductions; zeroed by the pre kernel)
  float* dk;          // fp32 BHND
  float* dv;          // fp32 BHND
  // -D_i = -sum_c dO_ic O_ic in the units of the scaled dS operand (see
  // exps): fp32 [B][H][n_pad], 0 past N
  float* delta;
  float* lse_log2;    // fp32 [B][H][n_pad]: L_i * log2(e) (+inf past N)
  void* q16;          // fp16 copies of q, k, v, dout scaled by 2^exps[t] (the
  void* k16;          // tensor-core operands)
  void* v16;
  void* do16;
  // kBwdAmaxBlocks x 4 partial maxima of |q|, |k|, |v|, |dout| (bf16
  // magnitude bits), reduced into the exponents e_q, e_k, e_v, e_do
  uint32_t* amax_part;
  int* exps;
  int B, H, N;
  int n_pad;          // N rounded up to a multiple of 128
  int causal;
  float scale;        // softmax scale
  float scale_log2;   // scale * log2(e)
  uint32_t* err;
  // packed variable-length mode when cu_q != nullptr (d = 128): q, o, dout, dq
  // [Tq][H][D]; k, v, dk, dv [Tk][Hkv][D]; lse [H][Tq]; N = the longest query
  // sequence, n_pad = N rounded up to 128, delta / lse_log2 [B][H][n_pad];
  // causal aligned to the bottom right
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int Hkv = 0, Tq = 0, Tk = 0, max_k = 0;
  long long n_q_elems = 0, n_k_elems = 0;   // elements of q (= dout) and of k (= v)
  // dropout on P (d = 128, [B, H, N, d] form), the forward's keep mask: drop_t
  // is the byte threshold, drop_scale = 256 / (256 - t)
  int dropout = 0;
  uint32_t drop_t = 0, seed_lo = 0, seed_hi = 0, drop_offset = 0;
  float drop_scale = 1.f;
  // d = 128, [B, H, N, d] form: (batch, head) slices per grid group (<= 0:
  // one group of all slices, key-block major over every head)
  int head_group = 0;
  // FP8 backward (fp8 = 1, [B, H, N, d] form): q, k, v are the FP8
  // forward's e4m3 codes (q, k of the rotated inputs) with fp32 scales sq, sk,
  // sv per 64-row block ([B][H][nsb]); the fp16 operand copies hold the codes
  // themselves (exact), and the block scales are folded in fp32
  int fp8 = 0;
  const float* sq = nullptr;
  const float* sk = nullptr;
  const float* sv = nullptr;
  int nsb = 0;
};

// Blocks of the backward's amax pass (the length of BwdArgs.amax_part / 4).
constexpr int kBwdAmaxBlocks = 148 * 4;

// tdq: fp32 view of dq, [BH][N][d], box 32 x 64, no swizzle (reduce-add target
// of the d = 128 main pass; unused for d = 64)
// ev_main_begin / ev_main_end (may be null): recorded on `stream` right before
// and right after the main pass, for timing that kernel alone.
template <int D>
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdArgs& a,
                       cudaStream_t stream, cudaEvent_t ev_main_begin = nullptr,
                       cudaEvent_t ev_main_end = nullptr);

// x[r][:] <- x[r][:] R^T in place for rows r < rows of two fp32 [rows][128]
// tensors x0, x1 (the FP8 backward's gradients of the rotated inputs back to
// the unrotated ones); a wait that gives up records its site in *err
cudaError_t launch_unrotate(float* x0, float* x1, const float* R, long long rows, int d,
                            uint32_t* err, cudaStream_t stream);

struct DecodeArgs {
  const void* q;            // bf16 [S][Hq][d]
  const void* k_cache;      // bf16 [P][Hkv][16][d]
  const void* v_cache;
  const int* block_table;   // int32 [S][max_blocks]
  int num_phys;             // physical blocks per cache (valid ids are [0, num_phys))
  const int* context_lens;  // int32 [S]
  void* o;                  // bf16 [S][Hq][d]
  float* lse;               // fp32 [S][Hq] or null
  float* part_o;            // fp32 [S][Hq][max_splits][d]
  float* part_l;            // fp32 [S][Hq][max_splits]
  unsigned int* counter;    // work-item counter (zeroed by the launcher)
  int num_seqs, Hq, Hkv, max_blocks, max_ctx, max_splits, split_blocks;
  int group;                // Hq / Hkv, 1 .. decode_max_group()
  int d;                    // head dimension, 64 or 128
  float scale_log2;
  uint32_t* err;
};

cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a,
                          cudaStream_t stream);

struct Fp8PrepArgs {
  const void* q;      // bf16 BHND
  const void* k;
  const void* v;
  const float* R;     // fp32 [d][d]
  uint8_t* q8;        // e4m3 BHND
  uint8_t* k8;
  uint8_t* v8;
  float* sq;          // fp32 [B][H][ceil(N/64)]
  float* sk;
  float* sv;
  int B, H, N;
  int d;              // head dim, 64 or 128
  uint32_t* err = nullptr;   // device error word (a bounded wait that gives up records its site)
};

cudaError_t launch_fp8_prepare(const Fp8PrepArgs& a, cudaStream_t stream);

struct Fp8FwdArgs {
  const float* sq;
  const float* sk;
  const float* sv;
  void* o;
  float* lse;
  int B, H, N;
  int d;              // head dim, 64 or 128
  int causal;
  int n_pairs;
  float scale_log2;
  uint32_t* err;
};

cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const Fp8FwdArgs& a, cudaStream_t stream);

cudaError_t launch_wait_probe(uint32_t* err, uint64_t limit_ns, cudaStream_t stream);

}  // namespace fa
