// api.cu — the extern "C" boundary declared in include/fa.h (and the
// profiling hook of include/fa_profiling.h): argument checks, TMA tensor-map
// encoding, workspace carving and kernel launches.
// No computation of the method happens here; every step runs in the kernels.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <math.h>
#include <string.h>

#include <atomic>

#include "fa.h"
#include "fa_profiling.h"
#include "kernels.h"
#include "prim.cuh"

namespace fa {
int decode_split_blocks();
int decode_max_group();
size_t decode_scratch_bytes();
cudaError_t decode_scratch_ptr(void** out);
}

namespace {

// Device error word: first bounded wait that gives up writes its site code.
__device__ uint32_t g_fa_error_word;

constexpr int kMaxDevices = 64;

uint32_t* error_word_ptr() {
  static std::atomic<uint32_t*> ptrs[kMaxDevices];   // racing first calls store the same value
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  uint32_t* w = ptrs[dev].load(std::memory_order_acquire);
  if (w == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fa_error_word) != cudaSuccess) return nullptr;
    w = static_cast<uint32_t*>(p);
    ptrs[dev].store(w, std::memory_order_release);
  }
  return w;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::atomic<EncodeTiledFn> cached{nullptr};
  EncodeTiledFn fn = cached.load(std::memory_order_acquire);
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &qr) == cudaSuccess &&
        qr == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
      cached.store(fn, std::memory_order_release);
    }
  }
  return fn;
}

// 3-D view [BH][N][d] of a BHND tensor, box (box_x elements, box_y rows, 1),
// 128-byte swizzle unless told otherwise, zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, int elem_bytes, int d,
              int n, int bh, uint32_t box_x, uint32_t box_y,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B, uint32_t box_z = 1) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(n),
                        static_cast<cuuint64_t>(bh)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem_bytes,
                           static_cast<cuuint64_t>(n) * d * elem_bytes};
  cuuint32_t box[3] = {box_x, box_y, box_z};
  cuuint32_t es[3] = {1, 1, 1};
  memset(m, 0, sizeof(*m));
  CUresult r = fn(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Events the next fa_bwd call of this thread records around its main pass.
thread_local cudaEvent_t g_bwd_ev_begin = nullptr;
thread_local cudaEvent_t g_bwd_ev_end = nullptr;

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

const float kLog2e = 1.4426950408889634f;

// Backward workspace part after D and L * log2(e): the amax partials of q, k,
// v, dout (4 words per amax block) and the four operand exponents.
constexpr size_t kStatsBytes =
    (4 * sizeof(uint32_t) * fa::kBwdAmaxBlocks + 4 * sizeof(int) + 255) / 256 * 256;

fa_status check_attn_dims(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > (1ll << 31) - 1) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H * N > (1ll << 31) - 1) return FA_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Grid grouping of the [B, H, N, d] forms: when the bytes the running CTAs
// stream per head (K and V in the forward; Q, dO and the fp32 dQ in the
// backward) exceed half of L2 over all heads, launch the heads in groups of 4
// so that those rows are shared in L2; otherwise (everything stays in L2) one
// group, which keeps the heaviest work first over all heads.
int head_group_for(int BH, int N, int d, int bytes_per_elem) {
  const double streamed = static_cast<double>(BH) * N * d * bytes_per_elem;
  return streamed > 64.0e6 ? 4 : 0;
}

// Dropout of the [B, H, N, d] forms: the byte threshold t = floor(256 p + 1/2)
// (t <= 255), the Philox key words and counter word 3, and 256 / (256 - t).
struct DropSpec {
  uint32_t t, seed_lo, seed_hi, offset;
  float scale;
};

bool drop_spec(float p, unsigned long long seed, unsigned int offset, DropSpec* out) {
  if (!(p >= 0.f)) return false;                      // also rejects NaN
  const double x = floor(256.0 * static_cast<double>(p) + 0.5);
  if (x > 255.0) return false;
  out->t = static_cast<uint32_t>(x);
  out->seed_lo = static_cast<uint32_t>(seed & 0xffffffffull);
  out->seed_hi = static_cast<uint32_t>(seed >> 32);
  out->offset = offset;
  out->scale = static_cast<float>(256.0 / (256.0 - x));
  return true;
}

fa_status fwd_dense(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int N, int d, int causal, void* stream, const DropSpec* drop) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  fa_status st = check_attn_dims(B, H, N, d);
  if (st != FA_OK) return st;
  uint32_t* err = error_word_ptr();
  if (err == nullptr) return FA_ERR_LAUNCH;
  CUtensorMap tq, tk, tv;
  const int bh = B * H;
  if (!make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, bh, 64, 128) ||
      !make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, bh, 64, 128) ||
      !make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, bh, 64, 128))
    return FA_ERR_LAUNCH;
  fa::FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.N = N;
  a.causal = causal ? 1 : 0;
  a.n_pairs = (N + 255) / 256;
  a.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  a.err = err;
  a.head_group = head_group_for(bh, N, d, 4);   // K and V, bf16
  if (drop != nullptr) {
    a.dropout = 1;
    a.drop_bias = (32768u - 128u * drop->t) * 0x00010001u;
    a.seed_lo = drop->seed_lo;
    a.seed_hi = drop->seed_hi;
    a.drop_offset = drop->offset;
    a.drop_scale = drop->scale;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = (d == 128) ? fa::launch_fwd<128>(tq, tk, tv, a, s)
                             : fa::launch_fwd<64>(tq, tk, tv, a, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

// The FP8 backward's extra inputs: the block scales of the e4m3 codes passed
// as q, k, v, and the rotation the codes of q and k were taken after.
struct Fp8Spec {
  const float* sq;
  const float* sk;
  const float* sv;
  const float* R;
};

fa_status bwd_dense(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dout, float* dq, float* dk, float* dv, void* workspace,
                    size_t ws_bytes, int B, int H, int N, int d, int causal, void* stream,
                    const DropSpec* drop, const Fp8Spec* f8 = nullptr) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  fa_status st = check_attn_dims(B, H, N, d);
  if (st != FA_OK) return st;
  if (f8 != nullptr && drop != nullptr) return FA_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned16(workspace) ||
      ws_bytes < fa_bwd_workspace_bytes(B, H, N, d))
    return FA_ERR_WORKSPACE;
  uint32_t* err = error_word_ptr();
  if (err == nullptr) return FA_ERR_LAUNCH;
  const int bh = B * H;
  const size_t n_pad = (static_cast<size_t>(N) + 127) / 128 * 128;
  const size_t prow = static_cast<size_t>(bh) * n_pad;
  const size_t tsz = round256(static_cast<size_t>(bh) * N * d * 2);
  char* w = static_cast<char*>(workspace);
  char* w16 = w + 2 * round256(prow * sizeof(float)) + kStatsBytes;
  void* q16 = w16;
  void* k16 = w16 + tsz;
  void* v16 = w16 + 2 * tsz;
  void* do16 = w16 + 3 * tsz;
  CUtensorMap tq, tk, tv, tdo, tdq;
  // steps over 128 queries at a time (128-row Q / dO boxes). The dQ reduce-add
  // boxes: 32 columns x 32 rows with the 128-byte swizzle (the drain writes a
  // query row per thread).
  const uint32_t qrows = 128;
  // K and V: the bf16 inputs themselves (the main pass converts them in shared
  // memory), or the fp16 copies of the FP8 backward's codes
  const bool kv16 = f8 != nullptr;
  const CUtensorMapDataType kv_dt = kv16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if (!make_map(&tq, q16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d, N, bh, 64, qrows) ||
      !make_map(&tk, kv16 ? k16 : k, kv_dt, 2, d, N, bh, 64, 128) ||
      !make_map(&tv, kv16 ? v16 : v, kv_dt, 2, d, N, bh, 64, 128) ||
      !make_map(&tdo, do16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d, N, bh, 64, qrows) ||
      !make_map(&tdq, dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, N, bh, 32, 32,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return FA_ERR_LAUNCH;
  fa::BwdArgs a;
  a.q16 = q16;
  a.k16 = k16;
  a.v16 = v16;
  a.do16 = do16;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.dout = dout;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.n_pad = static_cast<int>(n_pad);
  a.delta = static_cast<float*>(workspace);
  a.lse_log2 = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                        round256(prow * sizeof(float)));
  a.amax_part = reinterpret_cast<uint32_t*>(w + 2 * round256(prow * sizeof(float)));
  a.exps = reinterpret_cast<int*>(a.amax_part + 4 * fa::kBwdAmaxBlocks);
  a.B = B;
  a.H = H;
  a.N = N;
  a.causal = causal ? 1 : 0;
  a.scale = 1.0f / sqrtf(static_cast<float>(d));
  a.scale_log2 = a.scale * kLog2e;
  a.err = err;
  a.head_group = head_group_for(bh, N, d, 8);   // Q, dO fp16 and dQ fp32
  if (drop != nullptr) {
    a.dropout = 1;
    a.drop_t = drop->t;
    a.seed_lo = drop->seed_lo;
    a.seed_hi = drop->seed_hi;
    a.drop_offset = drop->offset;
    a.drop_scale = drop->scale;
  }
  if (f8 != nullptr) {
    a.fp8 = 1;
    a.sq = f8->sq;
    a.sk = f8->sk;
    a.sv = f8->sv;
    a.nsb = (N + 63) / 64;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t eb = g_bwd_ev_begin, ee = g_bwd_ev_end;
  g_bwd_ev_begin = g_bwd_ev_end = nullptr;     // one call consumes the pair
  cudaError_t e = (d == 128) ? fa::launch_bwd<128>(tq, tk, tv, tdo, tdq, a, s, eb, ee)
                             : fa::launch_bwd<64>(tq, tk, tv, tdo, tdq, a, s, eb, ee);
  if (e == cudaSuccess && f8 != nullptr) {
    // gradients of the rotated inputs -> of Q and K: dQ = dQ' R^T, dK = dK' R^T
    const long long rows = static_cast<long long>(bh) * N;
    e = fa::launch_unrotate(dq, dk, f8->R, rows, d, a.err, s);
  }
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

}  // namespace

namespace fa {
// the device error word of the current device, for kernels launched elsewhere
uint32_t* error_word_for_kv() { return error_word_ptr(); }
}  // namespace fa

extern "C" {

const char* fa_status_str(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_LAUNCH: return "FA_ERR_LAUNCH";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
  }
  return "FA_ERR_UNKNOWN";
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, int causal, void* stream) {
  return fwd_dense(q, k, v, o, lse, B, H, N, d, causal, stream, nullptr);
}

fa_status fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int N, int d, int causal, float p_drop, unsigned long long seed,
                         unsigned int offset, void* stream) {
  DropSpec ds;
  if (!drop_spec(p_drop, seed, offset, &ds)) return FA_ERR_INVALID_ARG;
  return fwd_dense(q, k, v, o, lse, B, H, N, d, causal, stream, &ds);
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                         const int* cu_seqlens_q, const int* cu_seqlens_k, int batch,
                         int max_seqlen_q, int total_q, int total_k, int H, int Hkv, int d,
                         int causal, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || lse == nullptr ||
      cu_seqlens_q == nullptr || cu_seqlens_k == nullptr)
    return FA_ERR_INVALID_ARG;
  if (batch < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || max_seqlen_q < 1 || total_q < 1 ||
      total_k < 1 || max_seqlen_q > total_q)
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long n_pairs = (static_cast<long long>(max_seqlen_q) + 255) / 256;
  if (static_cast<long long>(batch) * H * n_pairs > (1ll << 31) - 1 ||
      static_cast<long long>(total_q) * H > (1ll << 31) - 1 ||
      static_cast<long long>(total_k) * Hkv > (1ll << 31) - 1)
    return FA_ERR_UNSUPPORTED;
  uint32_t* err = error_word_ptr();
  if (err == nullptr) return FA_ERR_LAUNCH;
  // token-major views [T][heads][d]: x = head dim, y = head, z = token; a box is
  // 64 columns x 1 head x 128 tokens, the same 128 rows x 128 B in shared memory
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, H, total_q, 64, 1,
                CU_TENSOR_MAP_SWIZZLE_128B, 128) ||
      !make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, total_k, 64, 1,
                CU_TENSOR_MAP_SWIZZLE_128B, 128) ||
      !make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, total_k, 64, 1,
                CU_TENSOR_MAP_SWIZZLE_128B, 128))
    return FA_ERR_LAUNCH;
  fa::FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.B = batch;
  a.H = H;
  a.N = max_seqlen_q;
  a.causal = causal ? 1 : 0;
  a.n_pairs = static_cast<int>(n_pairs);
  a.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  a.err = err;
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.Hkv = Hkv;
  a.Tq = total_q;
  a.Tk = total_k;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = (d == 128) ? fa::launch_fwd<128>(tq, tk, tv, a, s)
                             : fa::launch_fwd<64>(tq, tk, tv, a, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

fa_status fa_paged_prefill(const void* q, const void* k_cache, const void* v_cache,
                           int num_phys_blocks, const int* block_table, int max_blocks_per_seq,
                           const int* cu_seqlens_q, const int* context_lens, void* o, float* lse,
                           int batch, int max_seqlen_q, int total_q, int Hq, int Hkv, int d,
                           int block_size, int causal, void* stream) {
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || block_table == nullptr ||
      cu_seqlens_q == nullptr || context_lens == nullptr || !aligned16(o) || lse == nullptr)
    return FA_ERR_INVALID_ARG;
  if (batch < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || max_seqlen_q < 1 || total_q < 1 ||
      max_seqlen_q > total_q || num_phys_blocks < 1 || max_blocks_per_seq < 1)
    return FA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || block_size != 16) return FA_ERR_UNSUPPORTED;
  const long long n_pairs = (static_cast<long long>(max_seqlen_q) + 255) / 256;
  if (static_cast<long long>(batch) * Hq * n_pairs > (1ll << 31) - 1 ||
      static_cast<long long>(total_q) * Hq > (1ll << 31) - 1 ||
      static_cast<long long>(num_phys_blocks) * Hkv * 16 > (1ll << 31) - 1 ||
      static_cast<long long>(max_blocks_per_seq) * 16 > (1ll << 31) - 1)
    return FA_ERR_UNSUPPORTED;
  uint32_t* err = error_word_ptr();
  if (err == nullptr) return FA_ERR_LAUNCH;
  // Q token-major [Tq][Hq][d]; the caches as [P * Hkv * 16][d] rows, boxes of
  // 64 columns x 16 rows (one physical block of one KV head)
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hq, total_q, 64, 1,
                CU_TENSOR_MAP_SWIZZLE_128B, 128) ||
      !make_map(&tk, k_cache, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d,
                num_phys_blocks * Hkv * 16, 1, 64, 16) ||
      !make_map(&tv, v_cache, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d,
                num_phys_blocks * Hkv * 16, 1, 64, 16))
    return FA_ERR_LAUNCH;
  fa::FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.B = batch;
  a.H = Hq;
  a.N = max_seqlen_q;
  a.causal = causal ? 1 : 0;
  a.n_pairs = static_cast<int>(n_pairs);
  a.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  a.err = err;
  a.cu_q = cu_seqlens_q;
  a.Hkv = Hkv;
  a.Tq = total_q;
  a.block_table = block_table;
  a.ctx = context_lens;
  a.max_blocks = max_blocks_per_seq;
  a.num_phys = num_phys_blocks;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = (d == 128) ? fa::launch_fwd<128>(tq, tk, tv, a, s)
                             : fa::launch_fwd<64>(tq, tk, tv, a, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

fa_status fa_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                              const unsigned char* block_mask, long long mask_bh_stride, int B,
                              int H, int N, int d, int causal, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      block_mask == nullptr || mask_bh_stride < 0)
    return FA_ERR_INVALID_ARG;
  fa_status st = check_attn_dims(B, H, N, d);
  if (st != FA_OK) return st;
  const long long nb = (static_cast<long long>(N) + 127) / 128;
  if (mask_bh_stride != 0 && mask_bh_stride < nb * nb) return FA_ERR_INVALID_ARG;
  if (nb > 512) return FA_ERR_UNSUPPORTED;            // N <= 65536 in this form
  uint32_t* err = error_word_ptr();
  if (err == nullptr) return FA_ERR_LAUNCH;
  CUtensorMap tq, tk, tv;
  const int bh = B * H;
  if (!make_map(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, bh, 64, 128) ||
      !make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, bh, 64, 128) ||
      !make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, N, bh, 64, 128))
    return FA_ERR_LAUNCH;
  fa::FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.N = N;
  a.causal = causal ? 1 : 0;
  a.n_pairs = (N + 255) / 256;
  a.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  a.err = err;
  // one group: with few key blocks kept per query block, K / V reuse is low
  // and the CTAs' work is uneven, so heaviest pair first over every head wins
  a.head_group = 0;
  a.block_mask = block_mask;
  a.mask_bh_stride = mask_bh_stride;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = (d == 128) ? fa::launch_fwd<128>(tq, tk, tv, a, s)
                             : fa::launch_fwd<64>(tq, tk, tv, a, s);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
  const size_t rows = static_cast<size_t>(B) * H * ((static_cast<size_t>(N) + 127) / 128 * 128);
  const size_t elems = static_cast<size_t>(B) * H * N * d;
  return 2 * round256(rows * sizeof(float)) + kStatsBytes + 4 * round256(elems * 2);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, float* dq, float* dk, float* dv, void* workspace,
                 size_t ws_bytes, int B, int H, int N, int d, int causal, void* stream) {
  return bwd_dense(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, H, N, d, causal,
                   stream, nullptr);
}

fa_status fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, float* dq, float* dk, float* dv,
                         void* workspace, size_t ws_bytes, int B, int H, int N, int d, int causal,
                         float p_drop, unsigned long long seed, unsigned int offset, void* stream) {
  DropSpec ds;
  if (!drop_spec(p_drop, seed, offset, &ds)) return FA_ERR_INVALID_ARG;
  return bwd_dense(q, k, v, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, H, N, d, causal,
                   stream, &ds);
}

fa_status fa_bwd_fp8(const void* q8, const void* k8, const void* v8, const float* sq,
                     const float* sk, const float* sv, const float* R, const void* o,
                     const float* lse, const void* dout, float* dq, float* dk, float* dv,
                     void* workspace, size_t ws_bytes, int B, int H, int N, int d, int causal,
                     void* stream) {
  if (!aligned16(sq) || !aligned16(sk) || !aligned16(sv) || !aligned16(R))
    return FA_ERR_INVALID_ARG;
  const Fp8Spec f8{sq, sk, sv, R};
  return bwd_dense(q8, k8, v8, o, lse, dout, dq, dk, dv, workspace, ws_bytes, B, H, N, d, causal,
                   stream, nullptr, &f8);
}

size_t fa_bwd_varlen_workspace_bytes(int batch, int max_seqlen_q, int total_q, int total_k, int H,
                                     int Hkv, int d) {
  if (batch < 1 || max_seqlen_q < 1 || total_q < 1 || total_k < 1 || H < 1 || Hkv < 1 || d < 1)
    return 0;
  const size_t rows = static_cast<size_t>(batch) * H *
                      ((static_cast<size_t>(max_seqlen_q) + 127) / 128 * 128);
  const size_t nq = static_cast<size_t>(total_q) * H * d, nk = static_cast<size_t>(total_k) * Hkv * d;
  return 2 * round256(rows * sizeof(float)) + kStatsBytes + 2 * round256(nq * 2) +
         2 * round256(nk * 2);
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o,
                        const float* lse, const void* dout, float* dq, float* dk, float* dv,
                        void* workspace, size_t ws_bytes, const int* cu_seqlens_q,
                        const int* cu_seqlens_k, int batch, int max_seqlen_q, int max_seqlen_k,
                        int total_q, int total_k, int H, int Hkv, int d, int causal,
                        void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || lse == nullptr ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      cu_seqlens_q == nullptr || cu_seqlens_k == nullptr)
    return FA_ERR_INVALID_ARG;
  if (batch < 1 || H < 1 || Hkv < 1 || H % Hkv != 0 || max_seqlen_q < 1 || max_seqlen_k < 1 ||
      total_q < 1 || total_k < 1 || max_seqlen_q > total_q || max_seqlen_k > total_k)
    return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long nkb = (static_cast<long long>(max_seqlen_k) + 127) / 128;
  if (static_cast<long long>(batch) * Hkv * nkb > (1ll << 31) - 1 ||
      static_cast<long long>(total_q) * H * d > (1ll << 40) ||
      static_cast<long long>(batch) * H * (max_seqlen_q + 127ll) > (1ll << 31) - 1)
    return FA_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned16(workspace) ||
      ws_bytes < fa_bwd_varlen_workspace_bytes(batch, max_seqlen_q, total_q, total_k, H, Hkv, d))
    return FA_ERR_WORKSPACE;
  uint32_t* err = error_word_ptr();
  if (err == nullptr) return FA_ERR_LAUNCH;
  const size_t n_pad = (static_cast<size_t>(max_seqlen_q) + 127) / 128 * 128;
  const size_t prow = static_cast<size_t>(batch) * H * n_pad;
  const size_t nq = static_cast<size_t>(total_q) * H * d, nk = static_cast<size_t>(total_k) * Hkv * d;
  char* w = static_cast<char*>(workspace);
  char* w16 = w + 2 * round256(prow * sizeof(float)) + kStatsBytes;
  void* q16 = w16;
  void* k16 = w16 + round256(nq * 2);
  void* v16 = w16 + round256(nq * 2) + round256(nk * 2);
  void* do16 = w16 + round256(nq * 2) + 2 * round256(nk * 2);
  // token-major views [T][heads][d]; Q / dO boxes of one step's 128 tokens,
  // K / V of 128, dQ reduce boxes as in fa_bwd
  CUtensorMap tq, tk, tv, tdo, tdq;
  const uint32_t qrows = 128;
  if (!make_map(&tq, q16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d, H, total_q, 64, 1,
                CU_TENSOR_MAP_SWIZZLE_128B, qrows) ||
      // K, V: the bf16 inputs (converted in shared memory by the main pass)
      !make_map(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, total_k, 64, 1,
                CU_TENSOR_MAP_SWIZZLE_128B, 128) ||
      !make_map(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d, Hkv, total_k, 64, 1,
                CU_TENSOR_MAP_SWIZZLE_128B, 128) ||
      !make_map(&tdo, do16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, d, H, total_q, 64, 1,
                CU_TENSOR_MAP_SWIZZLE_128B, qrows) ||
      !make_map(&tdq, dq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, d, H, total_q, 32, 1,
                CU_TENSOR_MAP_SWIZZLE_128B, 32))
    return FA_ERR_LAUNCH;
  fa::BwdArgs a;
  a.q16 = q16;
  a.k16 = k16;
  a.v16 = v16;
  a.do16 = do16;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.dout = dout;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.n_pad = static_cast<int>(n_pad);
  a.delta = static_cast<float*>(workspace);
  a.lse_log2 = reinterpret_cast<float*>(w + round256(prow * sizeof(float)));
  a.amax_part = reinterpret_cast<uint32_t*>(w + 2 * round256(prow * sizeof(float)));
  a.exps = reinterpret_cast<int*>(a.amax_part + 4 * fa::kBwdAmaxBlocks);
  a.B = batch;
  a.H = H;
  a.N = max_seqlen_q;
  a.causal = causal ? 1 : 0;
  a.scale = 1.0f / sqrtf(static_cast<float>(d));
  a.scale_log2 = a.scale * kLog2e;
  a.err = err;
  a.cu_q = cu_seqlens_q;
  a.cu_k = cu_seqlens_k;
  a.Hkv = Hkv;
  a.Tq = total_q;
  a.Tk = total_k;
  a.max_k = max_seqlen_k;
  a.n_q_elems = static_cast<long long>(nq);
  a.n_k_elems = static_cast<long long>(nk);
  cudaEvent_t eb = g_bwd_ev_begin, ee = g_bwd_ev_end;
  g_bwd_ev_begin = g_bwd_ev_end = nullptr;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = (d == 128) ? fa::launch_bwd<128>(tq, tk, tv, tdo, tdq, a, s, eb, ee)
                             : fa::launch_bwd<64>(tq, tk, tv, tdo, tdq, a, s, eb, ee);
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

size_t paged_attn_decode_workspace_bytes(int num_seqs, int Hq, int d, int max_ctx) {
  if (num_seqs < 1 || Hq < 1 || d < 1 || max_ctx < 1) return 0;
  const int sb = fa::decode_split_blocks();
  const size_t max_splits = ((static_cast<size_t>(max_ctx) + 15) / 16 + sb - 1) / sb;
  const size_t rows = static_cast<size_t>(num_seqs) * Hq * max_splits;
  return round256(rows * d * sizeof(float)) + round256(rows * sizeof(float)) + 256;
}

}  // extern "C"

namespace {
// The argument checks of the paged decode that do not involve the workspace
// (shared by paged_attn_decode and paged_attn_decode_noalloc).
fa_status decode_check(const void* q, const void* k_cache, const void* v_cache,
                       int num_phys_blocks, const int* block_table, int max_blocks_per_seq,
                       const int* context_lens, const void* o, const float* lse, int num_seqs,
                       int Hq, int Hkv, int d, int block_size, int max_ctx) {
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || block_table == nullptr ||
      context_lens == nullptr || !aligned16(o) || (lse != nullptr && !aligned16(lse)))
    return FA_ERR_INVALID_ARG;
  if (num_seqs < 1 || Hq < 1 || Hkv < 1 || d < 1 || block_size < 1 || max_ctx < 1 ||
      max_blocks_per_seq < 1 || num_phys_blocks < 1 || Hq % Hkv != 0)
    return FA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || block_size != 16 || Hq / Hkv > fa::decode_max_group())
    return FA_ERR_UNSUPPORTED;
  if (static_cast<long long>(max_blocks_per_seq) * 16 < max_ctx) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(num_phys_blocks) * Hkv * block_size > (1ll << 31) - 1)
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}
}  // namespace

extern "C" {

fa_status paged_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                            int num_phys_blocks, const int* block_table, int max_blocks_per_seq,
                            const int* context_lens, void* o, float* lse, int num_seqs, int Hq,
                            int Hkv, int d, int block_size, int max_ctx, void* workspace,
                            size_t ws_bytes, void* stream) {
  fa_status st = decode_check(q, k_cache, v_cache, num_phys_blocks, block_table,
                              max_blocks_per_seq, context_lens, o, lse, num_seqs, Hq, Hkv, d,
                              block_size, max_ctx);
  if (st != FA_OK) return st;
  const size_t need = paged_attn_decode_workspace_bytes(num_seqs, Hq, d, max_ctx);
  if (workspace == nullptr || !aligned16(workspace) || ws_bytes < need) return FA_ERR_WORKSPACE;
  uint32_t* err = error_word_ptr();
  if (err == nullptr) return FA_ERR_LAUNCH;
  const int sb = fa::decode_split_blocks();
  const int max_splits = ((max_ctx + 15) / 16 + sb - 1) / sb;
  if (max_splits > 65535) return FA_ERR_UNSUPPORTED;
  const size_t rows = static_cast<size_t>(num_seqs) * Hq * max_splits;
  fa::DecodeArgs a;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_table = block_table;
  a.num_phys = num_phys_blocks;
  a.context_lens = context_lens;
  a.o = o;
  a.lse = lse;
  a.part_o = static_cast<float*>(workspace);
  a.part_l = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                      round256(rows * d * sizeof(float)));
  a.counter = reinterpret_cast<unsigned int*>(static_cast<char*>(workspace) +
                                              round256(rows * d * sizeof(float)) +
                                              round256(rows * sizeof(float)));
  a.num_seqs = num_seqs;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.max_blocks = max_blocks_per_seq;
  a.max_ctx = max_ctx;
  a.max_splits = max_splits;
  a.split_blocks = sb;
  a.group = Hq / Hkv;
  a.d = d;
  a.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  a.err = err;
  // K / V caches as 2-D [blocks * Hkv * 16 rows][d] for 64-column, 16-row,
  // 128-byte-swizzled TMA boxes (one (block, kv head) slab = 2 boxes)
  CUtensorMap tk, tv;
  if (!make_map(&tk, k_cache, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d,
                num_phys_blocks * Hkv * block_size, 1, 64, block_size) ||
      !make_map(&tv, v_cache, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d,
                num_phys_blocks * Hkv * block_size, 1, 64, block_size))
    return FA_ERR_LAUNCH;
  cudaError_t e = fa::launch_decode(tk, tv, a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

fa_status paged_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                    int num_phys_blocks, const int* block_table,
                                    int max_blocks_per_seq, const int* context_lens, void* o,
                                    float* lse, int num_seqs, int Hq, int Hkv, int d,
                                    int block_size, int max_ctx, void* stream) {
  // Same checks as paged_attn_decode, then the library's own scratch array
  // stands in for the workspace (no allocation anywhere on this path).
  fa_status st = decode_check(q, k_cache, v_cache, num_phys_blocks, block_table,
                              max_blocks_per_seq, context_lens, o, lse, num_seqs, Hq, Hkv, d,
                              block_size, max_ctx);
  if (st != FA_OK) return st;
  const size_t need = paged_attn_decode_workspace_bytes(num_seqs, Hq, d, max_ctx);
  if (need > fa::decode_scratch_bytes()) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (fa::decode_scratch_ptr(&scratch) != cudaSuccess) return FA_ERR_LAUNCH;
  return paged_attn_decode(q, k_cache, v_cache, num_phys_blocks, block_table, max_blocks_per_seq,
                           context_lens, o, lse, num_seqs, Hq, Hkv, d, block_size, max_ctx,
                           scratch, fa::decode_scratch_bytes(), stream);
}

fa_status fa_fp8_prepare(const void* q, const void* k, const void* v, const float* R, void* q8,
                         void* k8, void* v8, float* sq, float* sk, float* sv, int B, int H,
                         int N, int d, void* stream) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(R) || !aligned16(q8) ||
      !aligned16(k8) || !aligned16(v8) || !aligned16(sq) || !aligned16(sk) || !aligned16(sv))
    return FA_ERR_INVALID_ARG;
  fa_status st = check_attn_dims(B, H, N, d);
  if (st != FA_OK) return st;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  fa::Fp8PrepArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.R = R;
  a.q8 = static_cast<uint8_t*>(q8);
  a.k8 = static_cast<uint8_t*>(k8);
  a.v8 = static_cast<uint8_t*>(v8);
  a.sq = sq;
  a.sk = sk;
  a.sv = sv;
  a.B = B;
  a.H = H;
  a.N = N;
  a.d = d;
  a.err = error_word_ptr();
  if (a.err == nullptr) return FA_ERR_LAUNCH;
  cudaError_t e = fa::launch_fp8_prepare(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* sq,
                     const float* sk, const float* sv, void* o, float* lse, int B, int H, int N,
                     int d, int causal, void* stream) {
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(sq) || !aligned16(sk) ||
      !aligned16(sv) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  fa_status st = check_attn_dims(B, H, N, d);
  if (st != FA_OK) return st;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  uint32_t* err = error_word_ptr();
  if (err == nullptr) return FA_ERR_LAUNCH;
  const int bh = B * H;
  CUtensorMap tq, tk, tv;
  // e4m3: one whole row (d bytes) per box row, swizzled over d bytes (the
  // kernel's MMA descriptors use the same pattern)
  const CUtensorMapSwizzle sw = d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if (!make_map(&tq, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, bh, d, 128, sw) ||
      !make_map(&tk, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, bh, d, 128, sw) ||
      !make_map(&tv, v8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, bh, d, 128, sw))
    return FA_ERR_LAUNCH;
  fa::Fp8FwdArgs a;
  a.sq = sq;
  a.sk = sk;
  a.sv = sv;
  a.o = o;
  a.lse = lse;
  a.B = B;
  a.H = H;
  a.N = N;
  a.d = d;
  a.causal = causal ? 1 : 0;
  a.n_pairs = (N + 255) / 256;
  a.scale_log2 = kLog2e / sqrtf(static_cast<float>(d));
  a.err = err;
  cudaError_t e = fa::launch_fwd_fp8(tq, tk, tv, a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

fa_status fa_bwd_time_main_pass(void* ev_begin, void* ev_end) {
  if ((ev_begin == nullptr) != (ev_end == nullptr)) return FA_ERR_INVALID_ARG;
  g_bwd_ev_begin = static_cast<cudaEvent_t>(ev_begin);
  g_bwd_ev_end = static_cast<cudaEvent_t>(ev_end);
  return FA_OK;
}

fa_status fa_last_device_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_LAUNCH;
  uint32_t word = 0;
  if (cudaMemcpyFromSymbol(&word, g_fa_error_word, sizeof(word)) != cudaSuccess)
    return FA_ERR_LAUNCH;
  if (word == 0) return FA_OK;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_fa_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return FA_ERR_LAUNCH;
  if (word & fa::kErrBadIndex) return FA_ERR_INVALID_ARG;
  if (word & fa::kErrRange) return FA_ERR_UNSUPPORTED;
  return FA_ERR_TIMEOUT;
}

fa_status fa_debug_wait_timeout(unsigned int timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 1000000u) return FA_ERR_INVALID_ARG;
  uint32_t* err = error_word_ptr();
  if (err == nullptr) return FA_ERR_LAUNCH;
  cudaError_t e = fa::launch_wait_probe(err, static_cast<uint64_t>(timeout_us) * 1000ull,
                                        static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : FA_ERR_LAUNCH;
}

}  // extern "C"

namespace fa {

namespace {
// One thread waits on a barrier that nothing arrives at; the bounded wait
// gives up after `limit_ns`, records the timeout and the kernel returns.
__global__ void wait_probe_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  abort_flag = 0;
  fence_mbar_init();
  mbar_wait(b, 0, err, 0x7f, &abort_flag, limit_ns);
}
}  // namespace

cudaError_t launch_wait_probe(uint32_t* err, uint64_t limit_ns, cudaStream_t stream) {
  wait_probe_kernel<<<1, 1, 0, stream>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace fa
