// bwd.cu — attention backward by recomputation for sm_100a.
//
// "Flash Attention 再学习" (jibinghu.github.io), backward: nothing N x N is
// stored by the forward; S and P are rebuilt tile by tile from Q, K and the
// per-row statistic. 91haoming.cn repost, "前向傳播改進": the statistic is the
// logsumexp L = m + log l alone, so P_ij = exp(scale * q_i.k_j - L_i).
// Same page, "并行化改進": the backward is parallel over K/V column blocks,
// and the gradient that crosses CTAs is accumulated with atomic adds. Here
// each CTA owns one 128-key block j (dK_j and dV_j stay on chip until the
// end) and the cross-CTA accumulation is dQ.
//
// Gradients (textbook softmax backward; the pages' formula images were lost):
//   D_i  = sum_c dO_ic O_ic                      (pre kernel; also zeroes dQ)
//   P    = exp(scale S - L),  S = Q K^T
//   dV_j += P^T dO_i,  dP = dO_i V_j^T,  dS = P o (dP - D_i)
//   dK_j += scale dS^T Q_i,  dQ_i += scale dS K_j   (fp32 reductions to HBM)
//
// Precision: the tensor-core operands of the backward are fp16 copies of the
// bf16 inputs, each tensor multiplied by a power of two picked from its
// largest magnitude so that its values sit inside fp16's range (an amax pass
// and the conversion pass, which copies Q and dO, run before the main pass;
// the main pass converts K and V itself; the factors are undone in fp32, see
// "operand scaling" below). P and dS, rounded to the operand type,
// keep 3 more mantissa bits than bf16 would give them. The scale of dS is
// chosen so that |dS| stays below 2^15 whenever L is the logsumexp of the
// scores; a dS beyond fp16's range (possible only with an inconsistent L) is
// recorded as FA_ERR_UNSUPPORTED.
//
// B200 mapping (one CTA per (batch*head, 128-key block), 512 threads; the
// kernel is bwd_ts_kernel below, templated on d = 64 / 128):
//   warp 0       TMA producer: K_j, V_j once; Q_i, dO_i, L_i, D_i per step of
//                128 queries, each refilled as soon as its last reader is done.
//   warp 1       TMEM allocation; lane 0 issues every tcgen05.mma: S^T, dP^T,
//                dV, dK and dQ (see "main pass on TMEM operands").
//   warps 4..11  thread = key row (TMEM lane), two warps per lane quarter,
//                one per half of the step's queries: first the in-place fp16
//                conversion of K and V, then per step P^T, written back into
//                TMEM as the A operand of dV, and dS, written into shared
//                memory for the dQ and dK products (d = 64: dS^T into TMEM
//                for dK); at the end the dK and dV rows.
//   warps 12..15 thread = query row: read the step's dQ tile out of TMEM and
//                add it to dQ in HBM with TMA tensor reduce-adds.
#include <climits>
#include <type_traits>

#include <atomic>
#include <utility>

#include "prim.cuh"
#include "kernels.h"

namespace fa {

// Pipeline trace (built only with -DFA_BWD_TRACE by exact_attention_102_b200.trace_bwd,
// never in libfa.so): CTA 0 of the [B, H, N, d] main pass records clock64
// stamps of its MMA-issuing thread, of one P / dS warp and of one drain warp.
#ifdef FA_BWD_TRACE
__device__ unsigned long long g_bwd_trace[3][8192];
#define FA_TRACE(row, tag)                                                             \
  do {                                                                                 \
    if (tr_on && tr_n[row] < 8192)                                                     \
      g_bwd_trace[row][tr_n[row]++] = (static_cast<unsigned long long>(clock64()) << 8) | (tag); \
  } while (0)
#else
#define FA_TRACE(row, tag) \
  do {                     \
  } while (0)
#endif

namespace {

enum : uint32_t {
  kSiteKV = 0x31, kSiteQE = 0x32, kSiteDE = 0x33, kSiteQF = 0x34, kSiteDF = 0x35, kSiteP = 0x36,
  kSiteDV = 0x37, kSiteDS = 0x38, kSiteDQF = 0x39, kSiteST = 0x3a, kSiteDPT = 0x3b,
  kSiteDSF = 0x3c, kSiteDQ = 0x3d, kSiteEnd = 0x3e, kSiteDrain = 0x3f, kSitePR = 0x40
};

// ------------------------------------------------------ operand scaling
// The tensor-core operands of the backward are fp16 (P and dS keep 3 more
// mantissa bits than bf16 would give them, and A and B of one MMA share a
// type). fp16 has 5 exponent bits against bf16's 8, so every input tensor X
// is first multiplied by a power of two 2^e_X chosen from its largest
// magnitude a_X = f 2^x (f in [0.5, 1)):
//   e_X = 14 - x,  so |X 2^e_X| < 2^14.
// A power-of-two factor changes no significant bit. A scaled element of
// magnitude >= 2^-17 is an fp16 value exactly (fp16 subnormals below that keep
// fewer than bf16's 8 bits), i.e. every element with |x| >= 2^-30 a_X converts
// exactly; a smaller one is rounded to a multiple of 2^(-24 - e_X), an error
// below 2^-38 a_X. The factors are undone in fp32, where they cost nothing:
//   S    = 2^-(e_q + e_k) S',             folded into scale * log2(e)
//   dP   = 2^-(e_do + e_v) dP'
//   dS'  = 2^sigma dS, sigma = e_do + e_v - 14 - log2(d), so that
//          dS' = P o (2^-(14 + log2 d) dP' - D'),  D' = 2^sigma D,
//          and |dS| <= P (|dP| + |D|) <= 2 d a_do a_v (O within V's range)
//          gives |dS'| < 2^15 (fp16 holds 65504)
//   dV   = 2^-e_do (P^T dO'),  dK = scale 2^-(sigma + e_q) (dS'^T Q'),
//   dQ   = scale 2^-(sigma + e_k) (dS' K').
// A tensor that is all zeros or holds a non-finite value keeps e_X = 0.
// bf16 magnitudes span 2^-133 .. 2^128, so e_X lies in [-114, 146].

// x * 2^n as two exact power-of-two multiplications (each factor a normal
// float); |n| is clamped to 252, beyond which the product of any finite
// nonzero fp32 value is 0 or infinite anyway.
struct Pow2 {
  float f1, f2;
};
__device__ __forceinline__ Pow2 pow2_pair(int n) {
  n = max(-252, min(252, n));
  const int n1 = n / 2, n2 = n - n1;
  return Pow2{__int_as_float((127 + n1) << 23), __int_as_float((127 + n2) << 23)};
}
__device__ __forceinline__ float mul_pow2(float x, Pow2 p) { return (x * p.f1) * p.f2; }
__device__ __forceinline__ float mul_pow2(float x, int n) { return mul_pow2(x, pow2_pair(n)); }

// e_X from the magnitude bits (0x0000 .. 0x7fff) of the largest |x|.
__device__ __forceinline__ int scale_exp(uint32_t mag) {
  if (mag == 0u || mag >= 0x7f80u) return 0;   // all zeros, or inf / NaN present
  int x;
  frexpf(__uint_as_float(mag << 16), &x);
  return 14 - x;
}

// 14 + log2(d) for the dS scale; d is 64 or 128
__device__ __forceinline__ int ds_shift(int D) { return D == 128 ? 21 : 20; }

// The four per-tensor maxima of |q|, |k|, |v|, |dout|: one partial per block
// (bf16 magnitude bits, compared as integers: for non-NaN values the order of
// the bits is the order of the magnitudes, and NaN sorts above infinity).
__global__ void __launch_bounds__(256) bwd_amax_kernel(BwdArgs a, long long q8, long long k8) {
  pdl_wait();                 // the inputs may come from the kernel before this one
  __shared__ uint32_t red[8][4];
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  uint32_t m[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    if (a.fp8 && t < 3) {
      // FP8 backward: the largest block scale of q, k, v (positive floats
      // compare as their bit patterns); the codes themselves need no scale
      const float* src = t == 0 ? a.sq : t == 1 ? a.sk : a.sv;
      const long long n = static_cast<long long>(a.B) * a.H * a.nsb;
      uint32_t mm = 0u;
      for (long long i = tid; i < n; i += stride) mm = max(mm, __float_as_uint(fabsf(src[i])));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mm = max(mm, __shfl_xor_sync(0xffffffffu, mm, off));
      m[t] = mm;
      continue;
    }
    const uint4* src = static_cast<const uint4*>(t == 0 ? a.q : t == 1 ? a.k : t == 2 ? a.v : a.dout);
    const long long n = (t == 0 || t == 3) ? q8 : k8;
    uint32_t mm = 0u;
    auto fold = [&](const uint4& u) {
      mm = __vmaxu2(mm, __vmaxu2(__vmaxu2(u.x & 0x7fff7fffu, u.y & 0x7fff7fffu),
                                 __vmaxu2(u.z & 0x7fff7fffu, u.w & 0x7fff7fffu)));
    };
    long long i = tid;
    for (; i + 3 * stride < n; i += 4 * stride) {    // four loads in flight per thread
      const uint4 u0 = src[i], u1 = src[i + stride], u2 = src[i + 2 * stride], u3 = src[i + 3 * stride];
      fold(u0);
      fold(u1);
      fold(u2);
      fold(u3);
    }
    for (; i < n; i += stride) fold(src[i]);
    mm = max(mm & 0xffffu, mm >> 16);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mm = max(mm, __shfl_xor_sync(0xffffffffu, mm, off));
    m[t] = mm;
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0)
    for (int t = 0; t < 4; ++t) red[w][t] = m[t];
  __syncthreads();
  if (threadIdx.x < 4) {
    uint32_t r = 0u;
    for (int i = 0; i < 8; ++i) r = max(r, red[i][threadIdx.x]);
    a.amax_part[blockIdx.x * 4 + threadIdx.x] = r;
  }
  pdl_trigger();              // this block's work is done: the next kernel may start
}

// Reduces the partial maxima into e_q, e_k, e_v, e_do (in shared memory).
__device__ __forceinline__ void load_exps(const BwdArgs& a, int (&e)[4]) {
  __shared__ uint32_t red[8][4];
  uint32_t m[4] = {0u, 0u, 0u, 0u};
  for (int i = threadIdx.x; i < kBwdAmaxBlocks; i += blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(a.amax_part)[i];
    m[0] = max(m[0], u.x);
    m[1] = max(m[1], u.y);
    m[2] = max(m[2], u.z);
    m[3] = max(m[3], u.w);
  }
#pragma unroll
  for (int t = 0; t < 4; ++t)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m[t] = max(m[t], __shfl_xor_sync(0xffffffffu, m[t], off));
  if ((threadIdx.x & 31) == 0)
    for (int t = 0; t < 4; ++t) red[threadIdx.x >> 5][t] = m[t];
  __syncthreads();
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    uint32_t r = 0u;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) r = max(r, red[i][t]);
    e[t] = scale_exp(r);
  }
}

// FP8 backward: the operands are the forward's e4m3 codes (exact fp16 values),
// the block scales are folded in fp32, and dO is scaled like the bf16 path.
// dS' = dS sq_i sk_j 2^tau is bounded like R22's dS':
//   |dS| <= 2 d max|dO| max|V|, max|V| <= 448 max(sv), so with
//   tau = e_do + 15 - ceil(log2(2 d 2^14 448 max(sq) max(sk) max(sv)))
//   |dS'| <= 2^15 (max|dO| 2^e_do < 2^14).
// exps[] then holds {tau, 0, 0, e_do}.
template <int D>
__device__ void fp8_convert(const BwdArgs& a, const int (&e)[4], long long q16) {
  // e[0..2]: scale_exp of the largest block scales' bit patterns is not what is
  // wanted here; recover the maxima from the partials directly
  __shared__ float smax[3];
  if (threadIdx.x < 3) {
    uint32_t r = 0u;
    for (int i = 0; i < kBwdAmaxBlocks; ++i) r = max(r, a.amax_part[i * 4 + threadIdx.x]);
    smax[threadIdx.x] = __uint_as_float(r);
  }
  __syncthreads();
  const int e_do = e[3];
  const float bound = 2.f * static_cast<float>(D) * 16384.f * 448.f;   // 2 d 2^14 448
  int c = 0;
  frexpf(bound * fmaxf(smax[0], 1e-30f) * fmaxf(smax[1], 1e-30f) * fmaxf(smax[2], 1e-30f), &c);
  const int tau = e_do + 15 - c;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    a.exps[0] = tau;
    a.exps[1] = 0;
    a.exps[2] = 0;
    a.exps[3] = e_do;
  }
  const Pow2 fdo = pow2_pair(e_do);
  // units of 16 bytes: e4m3 codes of q, k, v (16 codes -> 32 bytes of fp16),
  // then dO (8 bf16 -> 16 bytes of fp16)
  const long long c16 = q16 / 2;                    // 16-code units per tensor
  const long long total = 3 * c16 + q16;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    if (i < 3 * c16) {
      const int t = static_cast<int>(i / c16);
      const long long j = i - t * c16;
      const uint4 u = static_cast<const uint4*>(t == 0 ? a.q : t == 1 ? a.k : a.v)[j];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[8];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        asm("{\n\t.reg .b16 lo, hi;\n\t"
            "mov.b32 {lo, hi}, %2;\n\t"
            "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
            "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
            : "=r"(o[2 * cc]), "=r"(o[2 * cc + 1])
            : "r"(w[cc]));
      }
      uint4* dp = static_cast<uint4*>(t == 0 ? a.q16 : t == 1 ? a.k16 : a.v16) + 2 * j;
      dp[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dp[1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
      const long long j = i - 3 * c16;
      const uint4 u = static_cast<const uint4*>(a.dout)[j];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      uint32_t o[4];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
        o[cc] = pack_f16x2(mul_pow2(__uint_as_float(w[cc] << 16), fdo),
                           mul_pow2(__uint_as_float(w[cc] & 0xffff0000u), fdo));
      static_cast<uint4*>(a.do16)[j] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// Eight bf16 values (one 16-byte unit) -> eight fp16 values times 2^e.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4& u, Pow2 f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
  uint32_t o[4];
#pragma unroll
  for (int c = 0; c < 4; ++c)
    o[c] = pack_f16x2(mul_pow2(__uint_as_float(w[c] << 16), f),
                      mul_pow2(__uint_as_float(w[c] & 0xffff0000u), f));
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// ------------------------------------------------------- fp16 conversion
// q, dout (bf16) -> fp16 copies scaled by 2^e_X; 8 elements per thread per
// step, dout first (the amax pass reads it last, so its last rows may still
// be in L2). K and V are converted by the main pass itself, once per CTA, in
// shared memory. Block 0 publishes the exponents for the kernels that follow.
template <int D>
__global__ void __launch_bounds__(256) bwd_convert_kernel(BwdArgs a, long long q8, long long k8) {
  pdl_wait();                 // the amax partials
  int e[4];
  load_exps(a, e);
  if (a.fp8) {
    fp8_convert<D>(a, e, q8);
    return;
  }
  if (blockIdx.x == 0 && threadIdx.x < 4) a.exps[threadIdx.x] = e[threadIdx.x];
  const Pow2 f[4] = {pow2_pair(e[0]), pow2_pair(e[1]), pow2_pair(e[2]), pow2_pair(e[3])};
  (void)k8;
  const long long total = 2 * q8;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  // unit i: tensor (dout, then q) and offset
  auto locate = [&](long long i, int& t, long long& j) {
    t = i < q8 ? 3 : 0;
    j = i < q8 ? i : i - q8;
  };
  auto store = [&](int t, long long j, const uint4& u) {
    static_cast<uint4*>(t == 0 ? a.q16 : a.do16)[j] = bf16x8_to_f16x8(u, f[t]);
  };
  auto src = [&](int t) { return static_cast<const uint4*>(t == 0 ? a.q : a.dout); };
  long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  for (; i + 3 * stride < total; i += 4 * stride) {   // four loads in flight per thread
    int t[4];
    long long j[4];
    uint4 u[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      locate(i + r * stride, t[r], j[r]);
      u[r] = src(t[r])[j[r]];
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) store(t[r], j[r], u[r]);
  }
  for (; i < total; i += stride) {
    int t;
    long long j;
    locate(i, t, j);
    store(t, j, src(t)[j]);
  }
}

// ---------------------------------------------------------------- pre pass
// Per padded row (bh, n), n < n_pad = ceil(N/128)*128:
//   delta[bh][n] = -D'_n = -2^-(14 + log2 d) sum_c (dO_nc 2^e_do)(O_nc 2^e_v)
//                  (0 for n >= N)
//   Ll[bh][n]    = L_n * log2(e)     (+inf for n >= N, so P = 0 there)
// and dQ rows n < N are zeroed (dQ is accumulated by the main pass).
// A row is read by D / 8 lanes, 16 bytes of O and of dO each; a warp takes
// kPreGroups groups of 32 / (D / 8) rows at a time, with every load of the
// groups (L included) issued before the first reduction.
constexpr int kPreGroups = 4;
template <int D>
constexpr int pre_rows_per_warp() { return kPreGroups * 32 / (D / 8); }

template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(BwdArgs a) {
  pdl_wait();                 // the exponents of the conversion pass
  constexpr int LPR = D / 8;                       // lanes per row
  constexpr int RPG = 32 / LPR;                    // rows per group
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR;                      // 8-element slice of the row
  const long long rows = static_cast<long long>(a.B) * a.H * a.n_pad;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const bool packed = a.cu_q != nullptr;
  // FP8 backward: -D'' = -sum_c dO'_c O_c (O in its own units; the block
  // scales enter in the main pass)
  const Pow2 f_v = pow2_pair(a.fp8 ? 0 : a.exps[2]), f_do = pow2_pair(a.exps[3]);
  const float alpha = a.fp8 ? 1.f : __int_as_float((127 - ds_shift(D)) << 23);
  for (long long base = static_cast<long long>(warp) * (RPG * kPreGroups); base < rows;
       base += static_cast<long long>(nw) * (RPG * kPreGroups)) {
    long long rr[kPreGroups];
    int state[kPreGroups];                         // 0: past the rows, 1: padding row, 2: live
    uint4 ov[kPreGroups], gv[kPreGroups];
    float lv[kPreGroups];
#pragma unroll
    for (int u = 0; u < kPreGroups; ++u) {
      const long long pr = base + u * RPG + lane / LPR;
      state[u] = 0;
      rr[u] = 0;
      ov[u] = gv[u] = make_uint4(0u, 0u, 0u, 0u);
      lv[u] = 0.f;
      if (pr < rows) {
        const long long bh = pr / a.n_pad;
        const int n = static_cast<int>(pr - bh * a.n_pad);
        // query row n of this (batch, head): BHND row bh * N + n, or packed
        // token tq0 + n of head h (row (tq0 + n) * H + h; L at [h][tq0 + n])
        int len = a.N;
        long long r = bh * a.N + n, lr = r;
        if (packed) {
          const int b = static_cast<int>(bh / a.H), h = static_cast<int>(bh % a.H);
          const int tq0 = a.cu_q[b];
          len = a.cu_q[b + 1] - tq0;
          if (tq0 < 0 || len < 0 || len > a.N || tq0 + len > a.Tq) len = 0;   // reported by the main pass
          r = static_cast<long long>(tq0 + n) * a.H + h;
          lr = static_cast<long long>(h) * a.Tq + tq0 + n;
        }
        state[u] = n < len ? 2 : 1;
        rr[u] = r;
        if (state[u] == 2) {
          ov[u] = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.o) + r * D)[sub];
          gv[u] = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.dout) + r * D)[sub];
          if (sub == 0) lv[u] = a.lse[lr];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPreGroups; ++u) {
      const uint32_t o4[4] = {ov[u].x, ov[u].y, ov[u].z, ov[u].w};
      const uint32_t g4[4] = {gv[u].x, gv[u].y, gv[u].z, gv[u].w};
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc = fmaf(mul_pow2(__uint_as_float(o4[c] << 16), f_v),
                   mul_pow2(__uint_as_float(g4[c] << 16), f_do), acc);
        acc = fmaf(mul_pow2(__uint_as_float(o4[c] & 0xffff0000u), f_v),
                   mul_pow2(__uint_as_float(g4[c] & 0xffff0000u), f_do), acc);
      }
      // the row's lanes are LPR consecutive lanes: a butterfly inside them
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (state[u] == 0) continue;
      const long long pr = base + u * RPG + lane / LPR;
      if (sub == 0) {
        a.delta[pr] = state[u] == 2 ? -alpha * acc : 0.f;
        a.lse_log2[pr] = state[u] == 2 ? lv[u] * 1.4426950408889634f : INFINITY;
      }
      if (state[u] == 2) {
        float4* dq = reinterpret_cast<float4*>(a.dq + rr[u] * D);
        dq[sub] = make_float4(0.f, 0.f, 0.f, 0.f);
        dq[sub + LPR] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
}

// The fp32 factors that undo the operand scales in the main passes.
struct BwdScales {
  float c_s;        // scale * log2(e) * 2^-(e_q + e_k): S' -> log2-domain scores
  float alpha;      // 2^-(14 + log2 d): dP' -> the dS' units
  float dv;         // 2^-e_do (times 1 / keep probability with dropout)
  float dk;         // scale * 2^-(sigma + e_q)
  float dq1, dq2;   // dq1 * dq2 = scale * 2^-(sigma + e_k) (dq2 = 1 unless out of range)
};

template <int D>
__device__ __forceinline__ BwdScales bwd_scales(const BwdArgs& a) {
  const int e_q = a.exps[0], e_k = a.exps[1], e_v = a.exps[2], e_do = a.exps[3];
  const int sigma = e_do + e_v - ds_shift(D);
  BwdScales s;
  s.c_s = mul_pow2(a.scale_log2, -(e_q + e_k));
  s.alpha = __int_as_float((127 - ds_shift(D)) << 23);
  s.dv = mul_pow2(a.dropout ? a.drop_scale : 1.f, -e_do);
  s.dk = mul_pow2(a.scale, -(sigma + e_q));
  const int nq = -(sigma + e_k);
  if (nq >= -100 && nq <= 100) {
    s.dq1 = mul_pow2(a.scale, nq);
    s.dq2 = 1.f;
  } else {
    s.dq1 = mul_pow2(a.scale, nq / 2);
    s.dq2 = mul_pow2(1.f, nq - nq / 2);
  }
  return s;
}

// --------------------------------- main pass on TMEM operands, d = 64 / 128
// Same method, tiled around what the tensor core does fastest. Measured on
// this part: a tcgen05.mma with M = 128 and N = 64 costs about as long as
// one with N = 128, so every product here has N = 128 (d = 128) or N = d
// (d = 64), over steps of BQ = 128 queries:
//   S^T  = K_j Q_i^T      A = K_j  (d = 64: TMEM; d = 128: shared), B = Q_i
//   dP^T = V_j dO_i^T     A = V_j  (shared memory),                 B = dO_i
//   dV  += P^T dO_i       A = P^T  (TMEM, written over S^T),        B = dO_i
//   dK  += dS^T Q_i       A = dS^T (d = 64: TMEM, written over dP^T;
//                                   d = 128: shared, K-major),     B = Q_i
//   dQ   = dS K_j         A = dS   (shared, MN-major),              B = K_j (shared, MN-major)
// TMEM, d = 128: S^T/P^T [0,128)  dP^T, then dQ [128,256)  dV [256,384)
//                dK [384,512): 640 columns of state in 512, because dQ(i)
//                lands over dP^T(i) once the softmax-gradient warps have read
//                it, and dP^T(i+1) waits for the drain warps to have read dQ(i).
//      d = 64:   K [0,32)  S^T/P^T [64,192)  dP^T/dS^T [192,320)  dQ [320,384)
//                dV [384,448)  dK [448,512)
// One tcgen05 issuer executes in issue order, so a product may overwrite
// columns that the product issued just before it reads. Per step:
//   d = 64:  dK(i), dP^T(i+1), dV(i+1), S^T(i+2), dQ(i)
//   d = 128: dQ(i), second half of dK(i) [while the drain reads dQ(i)],
//            dP^T(i+1), dV(i+1), S^T(i+2), first half of dK(i+1) (once the
//            first 32-query chunk of each half of dS(i+1) is in)
// The d = 128 chain dP^T -> dS -> dQ -> drain -> dP^T bounds the step; the
// exp work of P(i+1) and the dK halves run beside it.
// Warps 4..11 (two per TMEM lane quarter, one per half of the step's queries)
// compute P and then dS for their half, 32 queries at a time; dS also goes to
// shared memory for the dQ product (d = 128: for dK too). Warps 12..15 drain dQ (thread = query
// row) through 32-column x 32-row fp32 boxes with the 128-byte swizzle (so the
// row-per-thread writes meet no bank conflicts), added to dQ in HBM by TMA
// tensor reduce-adds: d = 128, two boxes per warp, the four column chunks in
// two rounds; d = 64, one box, the two chunks in turn.
template <int D_>
struct BwdTs {
  static constexpr int D = D_;
  // d = 128 ("wide"): S^T, dP^T and dQ are N = 128 products over 128-query
  // steps; K and dS stay out of TMEM (S^T, dQ and dK read them from shared
  // memory) and dQ lands over the dP^T columns once the softmax-gradient
  // warps have read dP, so that 4 x 128 columns hold S^T, dP^T (then dQ), dV
  // and dK.
  static constexpr bool WIDE = D == 128;
  static constexpr int BK = 128;                 // keys per CTA
  static constexpr int BQ = 128;                 // queries per step
  static constexpr int HQ = BQ / 2;              // queries per half (one P / dS warp)
  static constexpr int NCH = HQ / 32;            // 32-query chunks per half
  static constexpr int KV_TILE = 128 * D * 2;    // K or V tile (D / 64 column chunks)
  static constexpr int KV_CHUNK = 128 * 128;
  static constexpr int Q_TILE = BQ * D * 2;      // Q or dO tile (D / 64 chunks of BQ rows)
  static constexpr int Q_CHUNK = BQ * 128;
  // Q / dO stages. d = 64: at least 3, because S^T(i+2) is issued (and waits
  // for its stage) before dQ(i), whose completion frees stage i. Wide: Q
  // takes 2 (Q_i is freed by dK(i), issued before S^T(i+2)) and dO one
  // buffer (dO_i is last read by dV(i), dO_i+1 first by dP^T(i+1), issued
  // after dK(i), dQ(i) and the drain of dQ(i)).
  static constexpr int NS = WIDE ? 2 : 3;
  static constexpr int NSG = WIDE ? 1 : NS;      // dO buffers
  static constexpr int DS_CHUNK = BK * 128;      // 64 queries of dS^T: one 128 B row per key
  static constexpr int DS_BYTES = BK * BQ * 2;   // dS^T fp16 [key][BQ queries]
  static constexpr int NDS = WIDE ? 1 : 2;       // dS buffers
  // dQ staging: [32 queries][32 columns] fp32 boxes with the 128-byte
  // swizzle, a query row per drain thread; wide, two per drain warp (the
  // four column chunks in two rounds), d = 64 one (its two chunks in turn).
  static constexpr int NBOX = WIDE ? 2 : 1;
  static constexpr int DQ_STAGE = NBOX * 32 * 32 * 4;
  // L log2(e) and -D' of a step: d = 64, one per stage, loaded with it;
  // wide, one buffer each, refilled once its last reader is done (L(i+1)
  // after P(i), D(i+1) after dS(i)), a step ahead of its next reader
  static constexpr int LD_BYTES = (WIDE ? 1 : NS) * BQ * 4;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + KV_TILE;
  static constexpr int Q_OFF = V_OFF + KV_TILE;
  static constexpr int DO_OFF = Q_OFF + NS * Q_TILE;
  static constexpr int DS_OFF = DO_OFF + NSG * Q_TILE;
  static constexpr int DQS_OFF = DS_OFF + NDS * DS_BYTES; // the drain warps' staging boxes
  static constexpr int L_OFF = DQS_OFF + 4 * DQ_STAGE;
  static constexpr int DL_OFF = L_OFF + LD_BYTES;
  static constexpr int BAR_OFF = DL_OFF + LD_BYTES;
  // B_FULL[s]: Q (d = 64: also dO, L and D) of the step in stage s landed.
  // B_STEP[s]: stage s is free again. d = 64: committed after the dQ product
  // of the step (the dS buffer and the dQ tile are then ready too); wide:
  // after its dK product.
  // B_DS: phase i completes when the 8 softmax-gradient warps have written
  // dS(i). B_DQF: phase i completes when the 4 drain warps have read dQ out of
  // TMEM (d = 64: dQ(i-1), so that dQ(i) may overwrite it; wide: dQ(i), so
  // that dP^T(i+1) may). Wide only: B_DQD, committed after dQ(i); B_GFULL,
  // dO of step i landed; B_DOF, committed after dV(i) (the dO buffer is free);
  // B_LFULL, B_DFULL: L and D of step i landed. B_DS0: the first 32-query
  // chunk of each half of dS(i) is in shared memory (queries 0-31 and 64-95),
  // so that dK(i) may start on them while the second chunks are computed.
  static constexpr int B_KV = 0, B_FULL = 1, B_STEP = B_FULL + NS;
  static constexpr int B_KT = B_STEP + NS, B_ST = B_KT + 1, B_DPT = B_ST + 1, B_P = B_DPT + 1;
  static constexpr int B_DS = B_P + 1, B_DQF = B_DS + 1, B_DQD = B_DQF + 1, B_GFULL = B_DQD + 1;
  static constexpr int B_DOF = B_GFULL + 1, B_LFULL = B_DOF + 1, B_DFULL = B_LFULL + 1;
  static constexpr int B_DS0 = B_DFULL + 1;
  static constexpr int B_KVC = B_DS0 + 1;       // K, V converted to fp16 in place (bf16 inputs)
  static constexpr int B_END = B_KVC + 1, B_DRAIN = B_END + 1, NBAR = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int SMEM_BYTES = MISC_OFF + 16 + 1024;
  // TMEM. Wide: S^T/P^T [0,128)  dP^T, then dQ [128,256)  dV [256,384)
  // dK [384,512). d = 64: K [0,32)  S^T/P^T [64,192)  dP^T/dS^T [192,320)
  // dQ [320,384)  dV [384,448)  dK [448,512).
  static constexpr uint32_t COL_K = 0, COL_S = WIDE ? 0 : 64, COL_DP = COL_S + BQ,
                            COL_DQ = WIDE ? COL_DP : COL_DP + BQ,
                            COL_DV = WIDE ? COL_DP + BQ : COL_DQ + 64, COL_DK = COL_DV + D;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 512;
};
static_assert(BwdTs<128>::SMEM_BYTES <= 232448, "d = 128 backward exceeds shared memory");
static_assert(BwdTs<64>::SMEM_BYTES <= 232448, "d = 64 backward exceeds shared memory");
static_assert(BwdTs<128>::COL_DK + 128 == 512 && BwdTs<64>::COL_DK + 64 == 512, "TMEM plan");
static_assert(BwdTs<64>::DQS_OFF % 1024 == 0 && BwdTs<128>::DQS_OFF % 1024 == 0,
              "swizzled staging boxes need 1024 B alignment");

constexpr int kOrderMaxB = 256;   // packed backward: sequences ordered by query length
static_assert(BwdTs<128>::DS_BYTES >= 4 * (kOrderMaxB + 1), "order list exceeds the dS buffer");

// TMEM column of the 16-query group kk of a packed fp16 [key][BQ queries]
// operand whose 32-query chunks start 32 columns apart (each chunk's 16
// packed columns sit over the first half of its own 32 fp32 columns).
__device__ __forceinline__ uint32_t half_col(int kk) {
  return static_cast<uint32_t>((kk >> 1) * 32 + (kk & 1) * 8);
}

// PACKED selects the packed variable-length form (BwdArgs.cu_q != nullptr) at
// compile time, so the [B, H, N, d] instantiation carries none of its indexing.
// DROP ([B, H, N, d] form only) applies the forward's dropout mask Z:
// dV = (P o Z)^T dO / q and dS = P o (Z o dP / q - D), q the keep probability.
// The keep bit of (query i, key j) is byte j % 16 of the Philox call
// (j / 16, i, bh, offset). The 16 lanes holding keys 16g .. 16g+15 need the
// same call per query, so each lane computes the calls of two of the 32
// queries of its chunk and the words reach the lanes that need them by one
// shuffle per element: the source lane of query 4b + c exposes, in round r,
// word (c + r) % 4, which is what a lane needing word w reads in the round
// with (w - r) % 4 = c.
// FP8 ([B, H, N, d] form, d = 128, no dropout) runs the FP8 forward's
// backward on its e4m3 codes (see fp8_convert): the score of (query i, key j)
// is sq_i sk_j (codes), dP = 2^-e_do sv_j (dO' codes), and dS goes to the
// operands as dS sq_i sk_j 2^tau, so dK_j = scale 2^-tau / sk_j (dS'^T q-codes)
// and dQ_i = scale 2^-tau / sq_i (dS' k-codes); sq of a 64-query block and
// sk, sv of a thread's key are one scale each.
template <int D, bool PACKED, bool DROP, bool FP8 = false>
__global__ void __launch_bounds__(512, 1)
bwd_ts_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
              const __grid_constant__ CUtensorMap tmDQ, BwdArgs a) {
  using C = BwdTs<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // The problem of this CTA: one 128-key block of Lk keys against Lq queries.
  // BHND: (batch, head) bh, TMA coordinates (row, bh). Packed: sequence b and
  // KV head hk; the CTA walks every query head of the group (their dK, dV
  // contributions add up in TMEM), TMA coordinates (head, token).
  constexpr bool packed = PACKED;
  int kb, bh = 0, b = 0, hk = 0, group = 1, Lq = a.N, Lk = a.N, tq0 = 0, tk0 = 0;
  if (packed) {
    // The key blocks of one (sequence, KV head) are adjacent in the grid, so
    // the CTAs running at the same time stream the same Q, dO rows and add
    // into the same dQ rows (shared in L2). Sequences come longest query range
    // first (the work of each of their CTAs), up to kOrderMaxB of them; beyond
    // that, batch order.
    const int nkb_all = (a.max_k + C::BK - 1) / C::BK;
    const int o = static_cast<int>(blockIdx.x) / nkb_all;
    kb = static_cast<int>(blockIdx.x) % nkb_all;
    hk = o % a.Hkv;
    b = o / a.Hkv;
    if (a.B <= kOrderMaxB) {
      int* qlen = reinterpret_cast<int*>(smem + C::DS_OFF);   // free until the first dS
      int* pick = qlen + kOrderMaxB;
      for (int s_ = threadIdx.x; s_ < a.B; s_ += blockDim.x) qlen[s_] = a.cu_q[s_ + 1] - a.cu_q[s_];
      if (threadIdx.x == 0) *pick = b;
      __syncthreads();
      for (int s_ = threadIdx.x; s_ < a.B; s_ += blockDim.x) {
        const int ls = qlen[s_];
        int r = 0;
        for (int u = 0; u < a.B; ++u) r += qlen[u] > ls || (qlen[u] == ls && u < s_);
        if (r == b) *pick = s_;
      }
      __syncthreads();
      b = *pick;
    }
    group = a.H / a.Hkv;
    tq0 = a.cu_q[b];
    tk0 = a.cu_k[b];
    Lq = a.cu_q[b + 1] - tq0;
    Lk = a.cu_k[b + 1] - tk0;
    if (tq0 < 0 || tk0 < 0 || Lq < 0 || Lk < 0 || Lq > a.N || tq0 + Lq > a.Tq || tk0 + Lk > a.Tk) {
      if (threadIdx.x == 0 && kb == 0) atomicCAS(a.err, 0u, kErrBadIndex + 2);
      Lq = 0;
      Lk = 0;
    }
  } else {
    // (batch, head) slices in groups of BwdArgs.head_group, key-block major
    // inside a group: the heaviest key blocks still come first within each
    // group, and the CTAs running at the same time cover few heads, so the Q,
    // dO and dQ rows they stream are shared in L2 (the host groups only when
    // those outgrow L2).
    const int BH = a.B * a.H;
    const int nkb_all = (a.N + C::BK - 1) / C::BK;
    const int G = a.head_group > 0 ? min(a.head_group, BH) : BH;
    const int g = static_cast<int>(blockIdx.x) / (G * nkb_all);
    const int gsize = min(G, BH - g * G);
    const int r = static_cast<int>(blockIdx.x) - g * G * nkb_all;
    kb = r / gsize;
    bh = g * G + r % gsize;
  }
  if (kb * C::BK >= Lk) return;                        // no keys in this block
  const int off = a.causal ? Lk - Lq : 0;              // causal: query i sees keys <= i + off
  const int nq = (Lq + C::BQ - 1) / C::BQ;
  const int i0 = a.causal ? max(0, kb * C::BK - off) / C::BQ : 0;  // first step seeing these keys
  const int n_steps = max(0, nq - i0);
  const int n_it = group * n_steps;                    // (query head, step) pairs
  // iteration it = (query head hk * group + it / n_steps, query step i0 + it % n_steps);
  // each role walks it in order and keeps the pair as counters (no division)
  struct Walk {
    int step, head;
  };
  auto walk_start = [&]() { return Walk{i0, hk * group}; };
  auto walk_next = [&](Walk& w) {
    if (++w.step == nq) {
      w.step = i0;
      ++w.head;
    }
  };
  if (n_it == 0) {                                      // keys no query sees: dK = dV = 0
    for (int i = threadIdx.x; i < C::BK * D / 4 * 2; i += blockDim.x) {
      const int which = i / (C::BK * D / 4), rem = i % (C::BK * D / 4);
      const int key = kb * C::BK + rem / (D / 4);
      if (key < Lk) {
        const size_t orow = packed ? (static_cast<size_t>(tk0 + key) * a.Hkv + hk) * D
                                   : (static_cast<size_t>(bh) * a.N + key) * D;
        reinterpret_cast<float4*>((which ? a.dk : a.dv) + orow)[rem % (D / 4)] =
            make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    return;
  }

  auto bar = [&](int i) -> uint32_t { return base + C::BAR_OFF + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
#ifdef FA_BWD_TRACE
  const bool tr_on = blockIdx.x == 0 && !PACKED && !DROP;
  int tr_n[3] = {0, 0, 0};
#endif

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_KV), 1);
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(C::B_FULL + s), 1);
      mbar_init(bar(C::B_STEP + s), 1);
    }
    mbar_init(bar(C::B_KT), 8);     // one arrival per softmax-gradient warp
    mbar_init(bar(C::B_ST), 1);
    mbar_init(bar(C::B_DPT), 1);
    mbar_init(bar(C::B_P), 8);
    mbar_init(bar(C::B_DS), 8);       // the 8 softmax-gradient warps
    mbar_init(bar(C::B_DQF), 4);      // the 4 drain warps
    mbar_init(bar(C::B_DQD), 1);
    mbar_init(bar(C::B_GFULL), 1);
    mbar_init(bar(C::B_DOF), 1);
    mbar_init(bar(C::B_LFULL), 1);
    mbar_init(bar(C::B_DFULL), 1);
    mbar_init(bar(C::B_DS0), 8);
    mbar_init(bar(C::B_KVC), 8);      // the 8 softmax-gradient warps
    mbar_init(bar(C::B_END), 1);
    mbar_init(bar(C::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the operand copies, D, L and the zeroed dQ of the passes before this one
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      tma_prefetch_desc(&tmDQ);
      mbar_arrive_expect_tx(bar(C::B_KV), 2 * C::KV_TILE);
      for (int c = 0; c < D / 64; ++c) {
        const int ky = packed ? hk : kb * C::BK, kz = packed ? tk0 + kb * C::BK : bh;
        tma_load_3d(base + C::K_OFF + c * C::KV_CHUNK, &tmK, bar(C::B_KV), c * 64, ky, kz);
        tma_load_3d(base + C::V_OFF + c * C::KV_CHUNK, &tmV, bar(C::B_KV), c * 64, ky, kz);
      }
      int issued = 0, g_issued = 0, l_issued = 0, d_issued = 0;
      Walk w = walk_start();
      for (int it = 0; it < n_it; ++it, walk_next(w)) {
        const int s = it % C::NS;
        const uint32_t ph = ((it / C::NS) & 1) ^ 1;
        const int row = w.step * C::BQ;
        const int hq = w.head;
        const size_t prow = (packed ? static_cast<size_t>(b) * a.H + hq : static_cast<size_t>(bh)) *
                                a.n_pad + row;                           // 256 B aligned
        const int qy = packed ? hq : row, qz = packed ? tq0 + row : bh;
        if (!mbar_wait(bar(C::B_STEP + s), ph, a.err, kSiteQE, abort_flag)) break;
        const uint32_t full = bar(C::B_FULL + s);
        if constexpr (C::WIDE) {
          mbar_arrive_expect_tx(full, C::Q_TILE);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(base + C::Q_OFF + s * C::Q_TILE + c * C::Q_CHUNK, &tmQ, full, c * 64, qy, qz);
          issued = it + 1;
          // dO_it into the one dO buffer once dV(it-1) has read dO_it-1
          if (it >= 1 && !mbar_wait(bar(C::B_DOF), (it - 1) & 1, a.err, kSiteQE, abort_flag)) break;
          mbar_arrive_expect_tx(bar(C::B_GFULL), C::Q_TILE);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(base + C::DO_OFF + c * C::Q_CHUNK, &tmDO, bar(C::B_GFULL), c * 64, qy, qz);
          g_issued = it + 1;
          // L_it once P(it-1) is done with the L buffer, D_it once dS(it-1)
          // is done with the D buffer
          if (it >= 1 && !mbar_wait(bar(C::B_P), (it - 1) & 1, a.err, kSiteQE, abort_flag)) break;
          mbar_arrive_expect_tx(bar(C::B_LFULL), C::BQ * 4);
          bulk_load(base + C::L_OFF, a.lse_log2 + prow, C::BQ * 4, bar(C::B_LFULL));
          l_issued = it + 1;
          if (it >= 1 && !mbar_wait(bar(C::B_DS), (it - 1) & 1, a.err, kSiteQE, abort_flag)) break;
          mbar_arrive_expect_tx(bar(C::B_DFULL), C::BQ * 4);
          bulk_load(base + C::DL_OFF, a.delta + prow, C::BQ * 4, bar(C::B_DFULL));
          d_issued = it + 1;
        } else {
          mbar_arrive_expect_tx(full, 2 * (C::Q_TILE + C::BQ * 4));
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(base + C::Q_OFF + s * C::Q_TILE + c * C::Q_CHUNK, &tmQ, full, c * 64, qy, qz);
          bulk_load(base + C::L_OFF + s * C::BQ * 4, a.lse_log2 + prow, C::BQ * 4, full);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(base + C::DO_OFF + s * C::Q_TILE + c * C::Q_CHUNK, &tmDO, full, c * 64, qy,
                        qz);
          bulk_load(base + C::DL_OFF + s * C::BQ * 4, a.delta + prow, C::BQ * 4, full);
          issued = it + 1;
        }
      }
      // no copy may still be in flight when the CTA exits
      for (int it = max(0, issued - C::NS); it < issued; ++it) {
        mbar_wait(bar(C::B_FULL + it % C::NS), (it / C::NS) & 1, a.err, kSiteDrain, nullptr,
                  200000000ull);
      }
      if (g_issued > 0)
        mbar_wait(bar(C::B_GFULL), (g_issued - 1) & 1, a.err, kSiteDrain, nullptr, 200000000ull);
      if (l_issued > 0)
        mbar_wait(bar(C::B_LFULL), (l_issued - 1) & 1, a.err, kSiteDrain, nullptr, 200000000ull);
      if (d_issued > 0)
        mbar_wait(bar(C::B_DFULL), (d_issued - 1) & 1, a.err, kSiteDrain, nullptr, 200000000ull);
      mbar_wait(bar(C::B_KV), 0, a.err, kSiteDrain, nullptr, 200000000ull);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, C::BQ, 0, 0, 0);   // S^T, dP^T: K-major operands
      constexpr uint32_t idKM = idesc_f16(128, D, 0, 0, 1);      // dV, dK: A tmem, B MN-major
      // dQ (M = BQ, N = d): A = dS and B = K, both MN-major
      constexpr uint32_t idQ = idesc_f16(128, D, 0, 1, 1);
      // descriptors of the fixed tiles and of stage / buffer 0; a tile at a
      // byte offset is the base descriptor plus offset / 16 (start-address field)
      const uint64_t dV = smem_desc_sw128(base + C::V_OFF, 16, 1024);            // V, K-major
      const uint64_t dKk = smem_desc_sw128(base + C::K_OFF, 16, 1024);           // K, K-major
      const uint64_t dKt = smem_desc_sw128(base + C::K_OFF, C::KV_CHUNK, 1024);  // K, MN-major
      const uint64_t dQk = smem_desc_sw128(base + C::Q_OFF, 16, 1024);           // Q, K-major
      const uint64_t dQm = smem_desc_sw128(base + C::Q_OFF, C::Q_CHUNK, 1024);   // Q, MN-major
      const uint64_t dGk = smem_desc_sw128(base + C::DO_OFF, 16, 1024);          // dO, K-major
      const uint64_t dGm = smem_desc_sw128(base + C::DO_OFF, C::Q_CHUNK, 1024);  // dO, MN-major
      // dS^T, MN-major over two 64-query blocks DS_CHUNK apart: the A operand
      // of dQ (M = 128)
      const uint64_t dDS = smem_desc_sw128(base + C::DS_OFF, C::DS_CHUNK, 1024);
      // the same dS buffer as the K-major A operand of dK (wide): a key row of
      // 128 bytes per 64-query block, the blocks DS_CHUNK apart
      const uint64_t dDSk = smem_desc_sw128(base + C::DS_OFF, 16, 1024);
      auto add = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (bytes >> 4); };
      // K and V as fp16 operands: the FP8 backward's copies of the codes come
      // in by TMA as they are; bf16 inputs are converted in shared memory first
      bool ok = mbar_wait(bar(FP8 ? C::B_KV : C::B_KVC), 0, a.err, kSiteKV, abort_flag);
      if constexpr (!C::WIDE) ok = ok && mbar_wait(bar(C::B_KT), 0, a.err, kSiteKV, abort_flag);
      auto issue_s = [&](int it) -> bool {
        const int s = it % C::NS;
        if (!mbar_wait(bar(C::B_FULL + s), (it / C::NS) & 1, a.err, kSiteQF, abort_flag))
          return false;
        tc_fence_after();
        const uint64_t q = add(dQk, s * C::Q_TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // K = d: chunk kk/4, 32 B steps inside it
          const uint32_t kb_off = (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32;
          if constexpr (C::WIDE)
            umma_f16_ss(tmem + C::COL_S, add(dKk, (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32),
                        add(q, kb_off), idS, kk > 0);
          else
            umma_f16_ts(tmem + C::COL_S, tmem + C::COL_K + kk * 8, add(q, kb_off), idS, kk > 0);
        }
        umma_commit(bar(C::B_ST));
        return true;
      };
      // dP^T(it). d = 64: stage it % NS was waited for by issue_s(it), issued
      // before; wide: dO_it has its own barrier
      auto issue_dp = [&](int it) -> bool {
        if constexpr (C::WIDE) {
          if (!mbar_wait(bar(C::B_GFULL), it & 1, a.err, kSiteQF, abort_flag)) return false;
          tc_fence_after();
        }
        const uint64_t g = add(dGk, (it % C::NSG) * C::Q_TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_f16_ss(tmem + C::COL_DP, add(dV, (kk >> 2) * C::KV_CHUNK + (kk & 3) * 32),
                      add(g, (kk >> 2) * C::Q_CHUNK + (kk & 3) * 32), idS, kk > 0);
        umma_commit(bar(C::B_DPT));
        return true;
      };
      // dV(it) += P^T(it) dO_it: after P(it) is in TMEM
      auto issue_dv = [&](int it) -> bool {
        if (!mbar_wait(bar(C::B_P), it & 1, a.err, kSiteP, abort_flag)) return false;
        tc_fence_after();
        const uint64_t gm = add(dGm, (it % C::NSG) * C::Q_TILE);
        const uint32_t acc0 = it > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < C::BQ / 16; ++kk)
          umma_f16_ts(tmem + C::COL_DV, tmem + C::COL_S + half_col(kk), add(gm, kk * 2048), idKM,
                      kk > 0 ? 1u : acc0);
        if constexpr (C::WIDE) umma_commit(bar(C::B_DOF));   // dO buffer free once dV(it) ran
        return true;
      };
      // d = 64: dK(it) += dS^T(it) Q_it after dS(it) is in TMEM (B_DS phase it)
      auto issue_dk = [&](int it) -> bool {
        if (!mbar_wait(bar(C::B_DS), it & 1, a.err, kSiteDS, abort_flag)) return false;
        tc_fence_after();
        const uint64_t qm = add(dQm, (it % C::NS) * C::Q_TILE);
        const uint32_t acc0 = it > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < C::BQ / 16; ++kk)
          umma_f16_ts(tmem + C::COL_DK, tmem + C::COL_DP + half_col(kk), add(qm, kk * 2048), idKM,
                      kk > 0 ? 1u : acc0);
        return true;
      };
      // wide: dK(it) += dS^T(it) Q_it with dS^T from shared memory, in two
      // halves: the 16-query groups of the halves' first chunks (0, 1, 4, 5)
      // after B_DS0, the others (2, 3, 6, 7) after B_DS
      auto issue_dk_half = [&](int it, int half) -> bool {
        if (!mbar_wait(bar(half ? C::B_DS : C::B_DS0), it & 1, a.err, kSiteDS, abort_flag))
          return false;
        tc_fence_after();
        const uint64_t qm = add(dQm, (it % C::NS) * C::Q_TILE);
        const uint64_t dsk = add(dDSk, (it % C::NDS) * C::DS_BYTES);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int kk = (g >> 1) * 4 + (g & 1) + 2 * half;
          umma_f16_ss(tmem + C::COL_DK, add(dsk, (kk >> 2) * C::DS_CHUNK + (kk & 3) * 32),
                      add(qm, kk * 2048), idKM, (half | g) > 0 || it > 0 ? 1u : 0u);
        }
        return true;
      };
      // dQ(it) over the 128 keys, B / A = dS(it) in buffer it % NDS
      auto issue_dq = [&](int it) {
        const uint64_t ds = add(dDS, (it % C::NDS) * C::DS_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk)
          umma_f16_ss(tmem + C::COL_DQ, add(ds, kk * 2048), add(dKt, kk * 2048), idQ,
                      kk > 0 ? 1u : 0u);
      };
      // Issue order: S(0), dP(0), dV(0), S(1), then per step it
      //   d = 64: dK(it), dP(it+1), dV(it+1), S(it+2), dQ(it)
      //   wide:   dQ(it), dK(it) second half, dP(it+1), dV(it+1), S(it+2),
      //           dK(it+1) first half
      // Each wait (P(it+1) before dV(it+1), dS(it) before dK(it) and dQ(it),
      // and, wide, the drain of dQ(it) before dP(it+1)) falls while products
      // issued before it are still running. In-order execution makes the
      // overwrites safe: S(it+2) comes after dV(it+1) (which reads P(it+1)
      // from the S columns); d = 64, dP(it+1) after dK(it) (which reads dS(it)
      // from the dP columns). Wide, dK reads dS from shared memory, so dQ(it)
      // may land over the dP columns as soon as the softmax-gradient warps
      // have read dP(it) (B_DS), and dK(it)'s second half runs while the
      // drain warps read dQ(it) out of TMEM. S(it+2) goes before the first
      // half of dK(it+1) (which waits for the first chunks of dS(it+1)), so
      // that the next scores are ready when the softmax-gradient warps are
      // done with dS(it+1)
      if (ok) {
        tc_fence_after();
        ok = issue_s(0) && issue_dp(0) && issue_dv(0);
        if constexpr (C::WIDE) ok = ok && issue_dk_half(0, 0);
        if (ok && n_it > 1) ok = issue_s(1);
      }
      for (int it = 0; it < n_it && ok; ++it) {
        const int s = it % C::NS;
        FA_TRACE(0, 1);
        if constexpr (C::WIDE) {
          // all of dS(it) in shared memory, dP(it) read out of TMEM
          ok = mbar_wait(bar(C::B_DS), it & 1, a.err, kSiteDS, abort_flag);
          if (!ok) break;
          tc_fence_after();
          issue_dq(it);
          umma_commit(bar(C::B_DQD));                // dQ(it) ready in TMEM
          FA_TRACE(0, 2);
          ok = issue_dk_half(it, 1);
          if (!ok) break;
          umma_commit(bar(C::B_STEP + s));           // stage s free once dK(it) has run
          FA_TRACE(0, 3);
          if (it + 1 < n_it) {
            // dP(it+1) overwrites dQ(it): after the drain warps have read it
            ok = mbar_wait(bar(C::B_DQF), it & 1, a.err, kSiteDQF, abort_flag);
            FA_TRACE(0, 4);
            if (!ok) break;
            tc_fence_after();
            ok = issue_dp(it + 1);
            ok = ok && issue_dv(it + 1);
            FA_TRACE(0, 5);
            if (ok && it + 2 < n_it) ok = issue_s(it + 2);
            ok = ok && issue_dk_half(it + 1, 0);
            FA_TRACE(0, 6);
            if (!ok) break;
          }
        } else {
          ok = issue_dk(it);
          FA_TRACE(0, 2);
          if (!ok) break;
          if (it + 1 < n_it) {
            FA_TRACE(0, 3);
            ok = issue_dp(it + 1);
            FA_TRACE(0, 4);
            ok = ok && issue_dv(it + 1);
            FA_TRACE(0, 5);
            if (ok && it + 2 < n_it) ok = issue_s(it + 2);
            FA_TRACE(0, 6);
            if (!ok) break;
          }
          // dQ_it, once dQ(it-1) has been drained (B_DQF phase it)
          ok = mbar_wait(bar(C::B_DQF), it & 1, a.err, kSiteDQF, abort_flag);
          FA_TRACE(0, 7);
          if (!ok) break;
          tc_fence_after();
          issue_dq(it);
          umma_commit(bar(C::B_STEP + s));  // step it complete: stage s, dS buffer, dQ tile
        }
        FA_TRACE(0, 8);
      }
      umma_commit(bar(C::B_END));
      umma_commit(bar(C::B_DRAIN));
      mbar_wait(bar(C::B_DRAIN), 0, a.err, kSiteDrain, nullptr, 200000000ull);
    }
  } else if (warp >= 4 && warp < 12) {
    // ---------- P^T and dS^T for one half of the step's queries (thread = key row)
    const int quarter = warp & 3;
    const int h = (warp - 4) >> 2;
    const int r = quarter * 32 + lane;
    const int key = kb * C::BK + r;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const BwdScales sc = bwd_scales<D>(a);
    const float sl2 = FP8 ? a.scale_log2 : sc.c_s;
    // FP8: the block scales of this thread's key, and 2^(tau - e_do)
    float f8_sk = 1.f, f8_sv = 1.f, f8_k0 = 1.f;
    if constexpr (FP8) {
      const int kblk = min(key / 64, a.nsb - 1);
      f8_sk = a.sk[static_cast<size_t>(bh) * a.nsb + kblk];
      f8_sv = a.sv[static_cast<size_t>(bh) * a.nsb + kblk];
      f8_k0 = mul_pow2(1.f, a.exps[0] - a.exps[3]);
    }
    bool ok = true;
    // bf16 K and V (TMA copies of the inputs) -> fp16 scaled by 2^e_K, 2^e_V,
    // in place: thread (r, h) converts the 16-byte units of K row r and V row
    // r that it reads below for the TMEM copy of K (d = 64: half h of the
    // row; d = 128: chunk h), which together cover both tiles
    constexpr int UNITS = D / 16;                     // 16-byte units per half row
    auto unit_addr = [&](int off, int u) -> uint8_t* {
      const int unit = (D == 128 ? 0 : UNITS * h) + u;
      return smem + off + (D == 128 ? h * C::KV_CHUNK : 0) + r * 128 + ((unit ^ (r & 7)) << 4);
    };
    if constexpr (!FP8 || !C::WIDE)
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_KV), 0, a.err, kSiteKV, abort_flag));
    if constexpr (!FP8) {
      if (ok) {
        const Pow2 fk = pow2_pair(a.exps[1]), fv = pow2_pair(a.exps[2]);
#pragma unroll
        for (int u = 0; u < UNITS; ++u) {
          uint4* pk = reinterpret_cast<uint4*>(unit_addr(C::K_OFF, u));
          uint4* pv = reinterpret_cast<uint4*>(unit_addr(C::V_OFF, u));
          *pk = bf16x8_to_f16x8(*pk, fk);
          *pv = bf16x8_to_f16x8(*pv, fv);
        }
        fence_async_smem();                           // for the tensor core's reads
        warp_arrive(bar(C::B_KVC));
      }
    }
    if (ok && !C::WIDE) {
      // K row r: the A operand of S^T, packed two fp16 per TMEM column like the
      // swizzled shared-memory row it comes from; half h copies head-dim
      // columns [D/2 h, D/2 h + D/2)
      uint32_t kr[UNITS * 4];
#pragma unroll
      for (int u = 0; u < UNITS; ++u) {
        const uint4 v = *reinterpret_cast<const uint4*>(unit_addr(C::K_OFF, u));
        kr[4 * u] = v.x;
        kr[4 * u + 1] = v.y;
        kr[4 * u + 2] = v.z;
        kr[4 * u + 3] = v.w;
      }
      if constexpr (D == 128)
        tmem_st32(tmem + lane_off + C::COL_K + 32 * h, kr);
      else
        tmem_st16(tmem + lane_off + C::COL_K + 16 * h, kr);
      tmem_st_wait();
      tc_fence_before();
      warp_arrive(bar(C::B_KT));
    }
    Walk wk = walk_start();
    // FP8: sq of this half's 64 queries (one scale block) in the next step,
    // loaded one step ahead (the [B, H, N, d] walk goes through consecutive
    // steps of one head)
    auto sq_of = [&](int step) {
      return __ldg(a.sq + static_cast<size_t>(bh) * a.nsb + min(2 * step + h, a.nsb - 1));
    };
    float f8_sq_next = FP8 ? sq_of(i0) : 1.f;
    for (int it = 0; it < n_it && ok; ++it, walk_next(wk)) {
      const int s = it % C::NS;
      const int buf = it % C::NDS;
      if (warp == 4 && lane == 0) FA_TRACE(1, 1);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_ST), it & 1, a.err, kSiteST, abort_flag));
      if (C::WIDE && ok)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_LFULL), it & 1, a.err, kSiteST, abort_flag));
      if (warp == 4 && lane == 0) FA_TRACE(1, 2);
      if (!ok) break;
      tc_fence_after();
      const float f8_sq = f8_sq_next;
      if constexpr (FP8)
        if (wk.step + 1 < nq) f8_sq_next = sq_of(wk.step + 1);
      uint32_t pk[C::NCH][16];                         // P^T, fp16 pairs of queries
      uint32_t zm[C::NCH];                             // bit e: (query qc + e, key) kept
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch) {
        const int qoff = C::HQ * h + 32 * ch;          // first query of this chunk in the step
        const int qh = wk.step * C::BQ + qoff;
        const float* Ls =
            reinterpret_cast<const float*>(smem + C::L_OFF + (C::WIDE ? 0 : s) * C::BQ * 4) + qoff;
        const uint32_t s_addr = tmem + lane_off + C::COL_S + qoff;
        const bool need_mask = (a.causal && key > qh + off) || key >= Lk || qh + 31 >= Lq;
        uint32_t sr[32];
        tmem_ld32(s_addr, sr);
        tmem_ld_wait();
        const float sl2s = FP8 ? sl2 * f8_sq * f8_sk : sl2;
        const uint64_t nsl2 = f2_pack(-sl2s, -sl2s);
        // queries qh + i, i in [lo, hi), see this key; the masked form runs only
        // in the steps where some lane of the warp has a masked query
        const int lo = a.causal ? key - off - qh : INT_MIN;
        const int hi = key < Lk ? Lq - qh : INT_MIN;
        auto p_loop = [&](auto masked) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 lv = *reinterpret_cast<const float4*>(Ls + e);
            // y = L - scale log2e S on packed pairs; P = 2^-y
            float y[4];
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), nsl2,
                             f2_pack(lv.x, lv.y)), y[0], y[1]);
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e + 2]), __uint_as_float(sr[e + 3])), nsl2,
                             f2_pack(lv.z, lv.w)), y[2], y[3]);
            float p[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              p[u] = ex2_approx(-y[u]);
              if constexpr (decltype(masked)::value) {
                if (e + u < lo || e + u >= hi) p[u] = 0.f;
              }
            }
            pk[ch][e / 2] = pack_f16x2(p[0], p[1]);
            pk[ch][e / 2 + 1] = pack_f16x2(p[2], p[3]);
          }
        };
        if (__any_sync(0xffffffffu, need_mask))
          p_loop(std::true_type{});
        else
          p_loop(std::false_type{});
        zm[ch] = 0xffffffffu;
        if constexpr (DROP) {
          const uint32_t g = lane & 15, jg = static_cast<uint32_t>(key) >> 4;
          uint32_t x[2][4];                            // x[c][r] = word (lane % 4 + r) % 4
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint4 w = philox4x32_10(jg, static_cast<uint32_t>(qh) + g + 16u * c,
                                          static_cast<uint32_t>(bh), a.drop_offset, a.seed_lo,
                                          a.seed_hi);
            const bool r1 = lane & 1, r2 = lane & 2;
            const uint32_t a0 = r1 ? w.y : w.x, a1 = r1 ? w.z : w.y, a2 = r1 ? w.w : w.z,
                           a3 = r1 ? w.x : w.w;
            x[c][0] = r2 ? a2 : a0;
            x[c][1] = r2 ? a3 : a1;
            x[c][2] = r2 ? a0 : a2;
            x[c][3] = r2 ? a1 : a3;
          }
          const int wsel = static_cast<int>(g >> 2);   // the word holding this key's byte
          const uint32_t sh = 8u * (lane & 3);         // its byte within the word
          const uint32_t keep_add = 256u - a.drop_t;   // byte + keep_add >= 256 iff kept
          uint32_t z = 0u;
#pragma unroll
          for (int bq = 0; bq < 8; ++bq) {
#pragma unroll
            for (int rr = 0; rr < 4; ++rr) {
              const int c = (wsel - rr) & 3;           // query 4 bq + c arrives in round rr
              const uint32_t y = __shfl_sync(0xffffffffu, x[bq >> 2][rr],
                                             static_cast<int>(lane & 16) | ((4 * bq) & 15) | c);
              z |= ((((y >> sh) & 0xffu) + keep_add) >> 8) << (4 * bq + c);
            }
          }
          zm[ch] = z;
        }
        uint32_t pz[16];                               // P o Z for the dV product
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pz[e] = DROP ? pk[ch][e] & ((((zm[ch] >> (2 * e)) & 3u) * 0x8001u & 0x10001u) * 0xffffu)
                       : pk[ch][e];
        tmem_st16(s_addr, pz);                         // over this chunk's own S^T columns
      }
      tmem_st_wait();
      tc_fence_before();
      warp_arrive(bar(C::B_P));
      if (warp == 4 && lane == 0) FA_TRACE(1, 3);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_DPT), it & 1, a.err, kSiteDPT, abort_flag));
      if (C::WIDE && ok)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_DFULL), it & 1, a.err, kSiteDPT, abort_flag));
      if (warp == 4 && lane == 0) FA_TRACE(1, 4);
      if (!ok) break;
      // the dS buffer: wide, dQ(it-1) has read it (it ran before dP(it), whose
      // completion was just seen); d = 64, wait for dQ(it-2)
      if (!C::WIDE && it >= 2) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_STEP + (it - 2) % C::NS),
                                               ((it - 2) / C::NS) & 1, a.err, kSiteDSF, abort_flag));
        if (!ok) break;
      }
      tc_fence_after();
      if (warp == 4 && lane == 0) FA_TRACE(1, 5);
      // alpha (2^-(14 + log2 d)) brings dP' to the units of dS'; with dropout
      // it also carries 1 / q
      const float ga = DROP ? sc.alpha * a.drop_scale : sc.alpha;
      // FP8: dS' = P o (2^(tau-e_do) sq sk) (sv dP' - D''); the D'' factor h
      const float f8_h = f8_k0 * f8_sq * f8_sk;
      const float gaf = FP8 ? f8_h * f8_sv : ga;
      const uint64_t ga2 = f2_pack(gaf, gaf), h2 = f2_pack(f8_h, f8_h);
      float ds_max = 0.f;
#pragma unroll
      for (int ch = 0; ch < C::NCH; ++ch) {
        const int qoff = C::HQ * h + 32 * ch;
        const float* Ds =
            reinterpret_cast<const float*>(smem + C::DL_OFF + (C::WIDE ? 0 : s) * C::BQ * 4) + qoff;
        const uint32_t dp_addr = tmem + lane_off + C::COL_DP + qoff;
        uint32_t dr[32];
        tmem_ld32(dp_addr, dr);
        tmem_ld_wait();
        uint32_t w[16];                                // dS^T, fp16 pairs of queries
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 dv4 = *reinterpret_cast<const float4*>(Ds + e);   // -D'
          uint64_t g01 = f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1]));
          uint64_t g23 = f2_pack(__uint_as_float(dr[e + 2]), __uint_as_float(dr[e + 3]));
          if constexpr (DROP) {                        // dP -> Z o dP
            auto z = [&](int i) { return dr[i] & (0u - ((zm[ch] >> i) & 1u)); };
            g01 = f2_pack(__uint_as_float(z(e)), __uint_as_float(z(e + 1)));
            g23 = f2_pack(__uint_as_float(z(e + 2)), __uint_as_float(z(e + 3)));
          }
          // dS' = P o (alpha dP' - D') on packed pairs
          uint64_t nd01 = f2_pack(dv4.x, dv4.y), nd23 = f2_pack(dv4.z, dv4.w);
          if constexpr (FP8) {
            nd01 = f2_mul(nd01, h2);
            nd23 = f2_mul(nd23, h2);
          }
          const uint64_t d01 = f2_fma(g01, ga2, nd01);
          const uint64_t d23 = f2_fma(g23, ga2, nd23);
          const uint32_t pa = pk[ch][e / 2], pb = pk[ch][e / 2 + 1];
          float ds[4];
          f2_unpack(f2_mul(f2_pack(f16_lo(pa), f16_hi(pa)), d01), ds[0], ds[1]);
          f2_unpack(f2_mul(f2_pack(f16_lo(pb), f16_hi(pb)), d23), ds[2], ds[3]);
          ds_max = fmax3(ds_max, fmax3(fabsf(ds[0]), fabsf(ds[1]), fabsf(ds[2])), fabsf(ds[3]));
          w[e / 2] = pack_f16x2(ds[0], ds[1]);
          w[e / 2 + 1] = pack_f16x2(ds[2], ds[3]);
        }
        // d = 64: the A operand of dK, over own dP^T columns (wide: dK reads
        // the shared-memory copy)
        if constexpr (!C::WIDE) tmem_st16(dp_addr, w);
        // shared memory copy for dQ (and, wide, dK): the chunk's 64 bytes of the
        // key's 128-byte row in its 64-query block, XOR-swizzled with (key row
        // % 8) like a TMA SWIZZLE_128B tile
        uint8_t* ds_row = smem + C::DS_OFF + buf * C::DS_BYTES + (qoff / 64) * C::DS_CHUNK + r * 128;
        const int unit0 = (qoff % 64) / 8;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4* dst = reinterpret_cast<uint4*>(ds_row + (((unit0 + u) ^ (r & 7)) << 4));
          *dst = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
        if (C::WIDE && ch == 0) {                      // first chunk in: dK may start on it
          fence_async_smem();
          tc_fence_before();
          warp_arrive(bar(C::B_DS0));
        }
      }
      if (!(ds_max < 65504.f)) atomicCAS(a.err, 0u, kErrRange + 2);
      tmem_st_wait();
      fence_async_smem();
      tc_fence_before();
      warp_arrive(bar(C::B_DS));
      if (warp == 4 && lane == 0) FA_TRACE(1, 6);
    }
    // ---- epilogue: dV rows (half 0) or dK rows (half 1), thread = key
    if (ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_END), 0, a.err, kSiteEnd, abort_flag));
      if (ok) {
        tc_fence_after();
        const size_t orow = packed ? (static_cast<size_t>(tk0 + key) * a.Hkv + hk) * D
                                   : (static_cast<size_t>(bh) * a.N + key) * D;
        const uint32_t src = tmem + lane_off + (h ? C::COL_DK : C::COL_DV);
        float* dst = (h ? a.dk : a.dv) + orow;
        float mul = h ? sc.dk : sc.dv;
        if constexpr (FP8)
          if (h) mul = mul_pow2(a.scale / f8_sk, -a.exps[0]);   // scale 2^-tau / sk
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(src + c * 32, v);
          tmem_ld_wait();
          if (key < Lk) {
            float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              d4[e] = make_float4(__uint_as_float(v[4 * e]) * mul, __uint_as_float(v[4 * e + 1]) * mul,
                                  __uint_as_float(v[4 * e + 2]) * mul,
                                  __uint_as_float(v[4 * e + 3]) * mul);
          }
        }
      }
    }
    tc_fence_before();
  } else if (warp >= 12) {
    // ------------------------------------------ dQ tile -> HBM via TMA reduce-add
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const BwdScales bs = bwd_scales<D>(a);
    float sc = bs.dq1, sc2 = bs.dq2;
    bool two = sc2 != 1.f;
    const Pow2 f8_tau = pow2_pair(FP8 ? -a.exps[0] : 0);
    if constexpr (C::WIDE) {
      // thread = query row (TMEM lane); the four 32-column chunks of its dQ
      // row go through this warp's two swizzled [32 queries][32 columns]
      // boxes in two rounds and are added to dQ by TMA reduce-adds. TMEM is
      // released once the second round's chunks are in registers.
      uint8_t* srow = smem + C::DQS_OFF + quarter * C::DQ_STAGE + lane * 128;
      const uint32_t stage_addr = base + C::DQS_OFF + quarter * C::DQ_STAGE;
      Walk wq = walk_start();
      // FP8: s_q of this warp's 32 query rows, loaded one step ahead (the
      // scale of the first column pair comes before the second pair's TMEM
      // read and the arrival that lets dP(it+1) start)
      auto sq_of_rows = [&](const Walk& w) {
        const int q = w.step * C::BQ + quarter * 32;
        return __ldg(a.sq + static_cast<size_t>(bh) * a.nsb + min(q / 64, a.nsb - 1));
      };
      float sq_next = 1.f;
      if constexpr (FP8)
        if (n_it > 0) sq_next = sq_of_rows(wq);
      for (int it = 0; it < n_it; ++it, walk_next(wq)) {
        const int qr = wq.step * C::BQ + quarter * 32;   // this warp's 32 query rows
        if (warp == 12 && lane == 0) FA_TRACE(2, 1);
        if (!__all_sync(0xffffffffu,
                        mbar_wait(bar(C::B_DQD), it & 1, a.err, kSiteDQ, abort_flag)))
          break;
        if (warp == 12 && lane == 0) FA_TRACE(2, 2);
        tc_fence_after();
        float m1 = sc, m2 = sc2;
        bool tw = two;
        if constexpr (FP8) {                         // scale 2^-tau / sq of these 32 queries
          const float sq = sq_next;
          if (it + 1 < n_it) {
            Walk wn = wq;
            walk_next(wn);
            sq_next = sq_of_rows(wn);
          }
          m1 = a.scale / sq * f8_tau.f1;
          m2 = f8_tau.f2;
          tw = true;
        }
        const bool inside = packed ? tq0 + qr < a.Tq : qr < a.N;   // box starts in the tensor
        auto scale_pair = [&](uint32_t (&v0)[32], uint32_t (&v1)[32]) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float f0 = __uint_as_float(v0[j]) * m1, f1 = __uint_as_float(v1[j]) * m1;
            v0[j] = __float_as_uint(tw ? f0 * m2 : f0);
            v1[j] = __float_as_uint(tw ? f1 * m2 : f1);
          }
        };
        auto stage_pair = [&](const uint32_t (&v0)[32], const uint32_t (&v1)[32]) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint32_t* v = c ? v1 : v0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<uint4*>(srow + c * 4096 + ((u ^ (lane & 7)) << 4)) =
                  make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
          }
        };
        auto reduce_pair = [&](int rd) {
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (inside) {
              for (int c = 0; c < 2; ++c) {
                const int x = 64 * rd + 32 * c;
                if (packed)
                  tma_reduce_add_3d(&tmDQ, stage_addr + c * 4096, x, wq.head, tq0 + qr);
                else
                  tma_reduce_add_3d(&tmDQ, stage_addr + c * 4096, x, qr, bh);
              }
            }
            bulk_commit_group();
          }
        };
        // columns [0, 64): out of TMEM, scaled, into the boxes (the previous
        // step's reduces have long read them)
        {
          uint32_t v0[32], v1[32];
          tmem_ld32(tmem + lane_off + C::COL_DQ, v0);
          tmem_ld32(tmem + lane_off + C::COL_DQ + 32, v1);
          tmem_ld_wait();
          scale_pair(v0, v1);
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          stage_pair(v0, v1);
        }
        // columns [64, 128) out of TMEM: dP(it+1) may now overwrite dQ(it);
        // then the first boxes go out and the second pair follows them
        {
          uint32_t v0[32], v1[32];
          tmem_ld32(tmem + lane_off + C::COL_DQ + 64, v0);
          tmem_ld32(tmem + lane_off + C::COL_DQ + 96, v1);
          tmem_ld_wait();
          tc_fence_before();
          warp_arrive(bar(C::B_DQF));
          if (warp == 12 && lane == 0) FA_TRACE(2, 3);
          reduce_pair(0);
          scale_pair(v0, v1);
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          stage_pair(v0, v1);
          reduce_pair(1);
        }
      }
      if (lane == 0) bulk_wait_all();
      tc_fence_before();
    } else {
      // d = 64: thread = query row, 64 head-dim columns; a [32 queries][32
      // columns] box per column half, 16-byte units XOR-swizzled with (row %
      // 8) as the 128-byte-swizzled tensor map reads them; the second half
      // waits until the first has been read out of the box
      uint8_t* srow = smem + C::DQS_OFF + quarter * C::DQ_STAGE + lane * 128;
      const uint32_t stage_addr = base + C::DQS_OFF + quarter * C::DQ_STAGE;
      warp_arrive(bar(C::B_DQF));                    // phase 0: no dQ(-1) to drain
      Walk wq = walk_start();
      for (int it = 0; it < n_it; ++it, walk_next(wq)) {
        const int qr = wq.step * C::BQ + quarter * 32;   // this warp's 32 query rows
        if (!__all_sync(0xffffffffu, mbar_wait(bar(C::B_STEP + it % C::NS), (it / C::NS) & 1,
                                                a.err, kSiteDQ, abort_flag)))
          break;
        tc_fence_after();
        uint32_t v0[32], v1[32];
        tmem_ld32(tmem + lane_off + C::COL_DQ, v0);
        tmem_ld32(tmem + lane_off + C::COL_DQ + 32, v1);
        tmem_ld_wait();
        tc_fence_before();
        warp_arrive(bar(C::B_DQF));                  // dQ(it) read: counts for phase it+1
        float m1 = sc, m2 = sc2;
        bool tw = two;
        if constexpr (FP8) {                         // scale 2^-tau / sq of this thread's row
          const float sq = __ldg(a.sq + static_cast<size_t>(bh) * a.nsb +
                                 min((qr + lane) / 64, a.nsb - 1));
          m1 = a.scale / sq * f8_tau.f1;
          m2 = f8_tau.f2;
          tw = true;
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float f0 = __uint_as_float(v0[j]) * m1, f1 = __uint_as_float(v1[j]) * m1;
          v0[j] = __float_as_uint(tw ? f0 * m2 : f0);   // factor outside one float's range
          v1[j] = __float_as_uint(tw ? f1 * m2 : f1);
        }
        const bool inside = packed ? tq0 + qr < a.Tq : qr < a.N;   // box starts in the tensor
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (lane == 0) bulk_wait_read_all();       // the box's previous reduce has read it
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint32_t* v = c ? v1 : v0;
            *reinterpret_cast<uint4*>(srow + ((u ^ (lane & 7)) << 4)) =
                make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            // rows past the tensor are skipped; in the packed form, rows past
            // this sequence add exact zeros (dS = 0 there) to the next one's dQ
            if (inside) {
              if (packed)
                tma_reduce_add_3d(&tmDQ, stage_addr, c * 32, wq.head, tq0 + qr);
              else
                tma_reduce_add_3d(&tmDQ, stage_addr, c * 32, qr, bh);
            }
            bulk_commit_group();
          }
        }
      }
      if (lane == 0) bulk_wait_all();
      tc_fence_before();
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace

template <int D>
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdArgs& a,
                       cudaStream_t stream, cudaEvent_t ev_main_begin, cudaEvent_t ev_main_end) {
  using C = BwdTs<D>;
  static std::atomic<bool> attr_set[64];   // per device; racing first calls both set it
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(bwd_ts_kernel<D, false, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_ts_kernel<D, true, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_ts_kernel<D, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(bwd_ts_kernel<D, false, false, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const long long rows = static_cast<long long>(a.B) * a.H * a.n_pad;
  const long long per_blk = 8LL * pre_rows_per_warp<D>();   // 8 warps per block
  const long long want = (rows + per_blk - 1) / per_blk;
  const int pre_blocks = static_cast<int>(want < 148 * 8 ? want : 148 * 8);
  const long long q8 = (a.cu_q ? a.n_q_elems : static_cast<long long>(a.B) * a.H * a.N * D) / 8;
  const long long k8 = (a.cu_q ? a.n_k_elems : static_cast<long long>(a.B) * a.H * a.N * D) / 8;
  const long long cwant = (2 * q8 + 2 * k8 + 255) / 256;
  const int cblocks = static_cast<int>(cwant < 148 * 8 ? cwant : 148 * 8);
  cudaError_t e = launch_pdl(bwd_amax_kernel, dim3(kBwdAmaxBlocks), dim3(256), 0, stream, a, q8, k8);
  if (e == cudaSuccess)
    e = launch_pdl(bwd_convert_kernel<D>, dim3(cblocks), dim3(256), 0, stream, a, q8, k8);
  if (e == cudaSuccess) e = launch_pdl(bwd_pre_kernel<D>, dim3(pre_blocks), dim3(256), 0, stream, a);
  if (e != cudaSuccess) return e;
  const int nk = ((a.cu_q ? a.max_k : a.N) + C::BK - 1) / C::BK;
  const int per_block = a.cu_q ? a.B * a.Hkv : a.B * a.H;   // CTAs per key block
  if (ev_main_begin != nullptr) cudaEventRecord(ev_main_begin, stream);
  {
    void (*k)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, BwdArgs) =
        a.fp8 ? bwd_ts_kernel<D, false, false, true>
              : a.cu_q ? bwd_ts_kernel<D, true, false>
                       : a.dropout ? bwd_ts_kernel<D, false, true> : bwd_ts_kernel<D, false, false>;
    e = launch_pdl(k, dim3(nk * per_block), dim3(C::THREADS), C::SMEM_BYTES, stream, tq, tk, tv, tdo,
                   tdq, a);
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (ev_main_end != nullptr) cudaEventRecord(ev_main_end, stream);
  return e;
}

namespace {
// In place x[r][:] <- x[r][:] R^T, d = 128, for two tensors of `rows` rows
// each (the FP8 backward's dQ' and dK'), on the tensor core. Every fp32
// operand v is split into bf16 terms hi = bf16(v), lo = bf16(v - hi), and the
// product is hi_x hi_R + lo_x hi_R + hi_x lo_R with fp32 accumulation; the
// dropped lo_x lo_R and the rounding of the lo terms leave a relative error
// near 2^-16 of sum_e |x_e| |R_ce| per output.
//
// One tile = 128 rows. A (128 rows x K = 128) is the split x tile in TMEM,
// written by the threads (two bf16 per column); B is the split R in shared
// memory, K-major with the 128-byte swizzle (B row n = R row n, so
// D[m][n] = sum_e x[m][e] R[n][e]); D is the fp32 accumulator in TMEM.
// 8 warps: warp w reaches TMEM lanes 32 (w % 4) .. + 31 and takes head-dim
// half w / 4 of the loads and of the stores, both in the 16 x 256 bit TMEM
// shape, so that 4 neighbouring threads cover 64 (load) or 32 (store)
// contiguous bytes of one row. Two CTAs per SM (64 KB of shared memory and
// 256 TMEM columns each): one CTA's loads overlap the other's products, and
// each CTA loads its next tile while its own products run.
constexpr int kRotThreads = 256;
// R hi, R lo, alignment and the barrier take 66.6 KB; the request is 80 KB so
// that a third CTA (which would wait for TMEM columns) never shares an SM
constexpr int kRotSmem = 80 * 1024;
constexpr uint32_t kRotCols = 256;     // accumulator [0, 128), x hi [128, 192), x lo [192, 256)
constexpr uint32_t kSiteRot = 0x41;

__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(a, b);
  lo = pack_bf16x2(a - __uint_as_float(hi << 16), b - __uint_as_float(hi & 0xffff0000u));
}

__global__ void __launch_bounds__(kRotThreads, 2) unrotate_kernel(float* x0, float* x1,
                                                                   const float* __restrict__ R,
                                                                   long long rows, uint32_t* err) {
  extern __shared__ uint8_t rot_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rot_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(sm);
  const uint32_t bar = sbase + 65536;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + 65536 + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + 65536 + 16);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // R -> bf16 hi / lo, K-major, 128-byte swizzle: K chunk e / 64 at 16 KB
  // steps, row c at c * 128 B, 16-byte unit u of the row at unit u ^ (c % 8)
  for (int u = threadIdx.x; u < 128 * 16; u += kRotThreads) {
    const int c = u >> 4, e0 = (u & 15) * 8;
    const float4 a = __ldg(reinterpret_cast<const float4*>(R + c * 128 + e0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(R + c * 128 + e0 + 4));
    uint4 h, l;
    split_bf16x2(a.x, a.y, h.x, l.x);
    split_bf16x2(a.z, a.w, h.y, l.y);
    split_bf16x2(b.x, b.y, h.z, l.z);
    split_bf16x2(b.z, b.w, h.w, l.w);
    const uint32_t off = (e0 >> 6) * 16384 + c * 128 + ((((e0 & 63) >> 3) ^ (c & 7)) << 4);
    *reinterpret_cast<uint4*>(sm + off) = h;
    *reinterpret_cast<uint4*>(sm + 32768 + off) = l;
  }
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), kRotCols);
    tmem_relinquish();
  }
  fence_async_smem();     // R, written by the threads, seen by the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const long long tiles_per = (rows + 127) / 128, tiles = 2 * tiles_per;
  const int q = warp & 3, hh = warp >> 2, r_in = lane >> 2, cq = lane & 3;
  const uint32_t id = idesc_f16(128, 128, 1, 0, 0);
  const uint64_t dRh = smem_desc_sw128(sbase, 16, 1024);
  const uint64_t dRl = smem_desc_sw128(sbase + 32768, 16, 1024);
  auto add = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (bytes >> 4); };

  // this thread's part of a tile: rows 32 q + 16 i + 8 s + r_in (i, s in
  // {0, 1}); K groups j = 4 hh + g (g < 4), elements 16 j + 4 cq .. + 3
  float4 xv[2][2][4];
  auto load = [&](long long t) {
    const float* X = t < tiles_per ? x0 : x1;
    const long long r0 = (t < tiles_per ? t : t - tiles_per) * 128;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int s2 = 0; s2 < 2; ++s2) {
        const long long row = r0 + 32 * q + 16 * i + 8 * s2 + r_in;
        const float4* src = reinterpret_cast<const float4*>(X + row * 128 + 64 * hh + 4 * cq);
#pragma unroll
        for (int g = 0; g < 4; ++g)
          xv[i][s2][g] = row < rows ? __ldcs(src + 4 * g) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
  };

  long long t = blockIdx.x;
  if (t < tiles) load(t);
  uint32_t phase = 0;
  for (; t < tiles; t += gridDim.x) {
    // split x into TMEM columns 128 + (K group) * 8 (hi) and 192 + .. (lo)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      uint32_t hi[16], lo[16];
#pragma unroll
      for (int g = 0; g < 4; ++g)
#pragma unroll
        for (int s2 = 0; s2 < 2; ++s2) {
          const float4 v = xv[i][s2][g];
          split_bf16x2(v.x, v.y, hi[4 * g + 2 * s2], lo[4 * g + 2 * s2]);
          split_bf16x2(v.z, v.w, hi[4 * g + 2 * s2 + 1], lo[4 * g + 2 * s2 + 1]);
        }
      const uint32_t ta = tmem + (static_cast<uint32_t>(32 * q + 16 * i) << 16) + 32 * hh;
      tmem_st_16x256b_x4(ta + 128, hi);
      tmem_st_16x256b_x4(ta + 192, lo);
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_fence_after();
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        const uint32_t a_col = p == 1 ? 192 : 128;
        const uint64_t b = p == 2 ? dRl : dRh;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16_ts(tmem, tmem + a_col + 8 * kk, add(b, (kk >> 2) * 16384 + (kk & 3) * 32), id,
                      (p | kk) != 0);
      }
      umma_commit(bar);
    }
    const long long cur = t;
    if (t + gridDim.x < tiles) load(t + gridDim.x);    // next tile, while the products run
    const bool ok = mbar_wait(bar, phase, err, kSiteRot, abort_flag);
    if (__syncthreads_or(!ok)) break;      // every thread leaves the loop together
    phase ^= 1;
    tc_fence_after();
    float* X = cur < tiles_per ? x0 : x1;
    const long long r0 = (cur < tiles_per ? cur : cur - tiles_per) * 128;
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
      const int i = c4 >> 1, half = c4 & 1;
      uint32_t v[16];
      tmem_ld_16x256b_x4(
          tmem + (static_cast<uint32_t>(32 * q + 16 * i) << 16) + 64 * hh + 32 * half, v);
      tmem_ld_wait();
      const long long ra = r0 + 32 * q + 16 * i + r_in, rb = ra + 8;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int col = 64 * hh + 32 * half + 8 * g + 2 * cq;
        if (ra < rows)
          __stcs(reinterpret_cast<float2*>(X + ra * 128 + col),
                 make_float2(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1])));
        if (rb < rows)
          __stcs(reinterpret_cast<float2*>(X + rb * 128 + col),
                 make_float2(__uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3])));
      }
    }
    tc_fence_before();
  }
  // a wait that gave up leaves products possibly in flight: wait for them
  // (bounded) before the columns are freed
  if (*abort_flag) mbar_wait(bar, phase, nullptr, kSiteRot, nullptr, 100000000ull);
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kRotCols);
  }
}
}  // namespace

namespace {
// d = 64: x[r][:] <- x[r][:] R^T in fp32 on the CUDA cores (64 x 64 multiply-
// adds per row), in place, 64-row tiles of both tensors. Rt[e][c] = R[c][e]
// in shared memory; thread t computes rows 4 (t / 16) .. + 3, columns
// 4 (t % 16) .. + 3.
constexpr int kRot64Smem = 2 * 64 * 64 * 4;
__global__ void __launch_bounds__(256) unrotate64_kernel(float* x0, float* x1,
                                                        const float* __restrict__ R, long long rows) {
  extern __shared__ __align__(16) float rs[];
  float* Rt = rs;
  float* xs = rs + 64 * 64;
  for (int i = threadIdx.x; i < 64 * 64; i += 256) Rt[(i % 64) * 64 + i / 64] = R[i];
  const int r4 = (threadIdx.x >> 4) * 4, c4 = (threadIdx.x & 15) * 4;
  const long long tiles_per = (rows + 63) / 64;
  for (long long t = blockIdx.x; t < 2 * tiles_per; t += gridDim.x) {
    float* X = t < tiles_per ? x0 : x1;
    const long long r0 = (t < tiles_per ? t : t - tiles_per) * 64;
    const int nr = static_cast<int>(min(64ll, rows - r0));
    __syncthreads();                               // Rt written / previous tile read
    for (int i = threadIdx.x; i < 64 * 16; i += 256)
      reinterpret_cast<float4*>(xs)[i] = i < nr * 16 ? reinterpret_cast<const float4*>(X + r0 * 64)[i]
                                                     : make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    float y[4][4] = {};
#pragma unroll 8
    for (int e = 0; e < 64; ++e) {
      const float4 rv = *reinterpret_cast<const float4*>(Rt + e * 64 + c4);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float xe = xs[(r4 + i) * 64 + e];
        y[i][0] = fmaf(xe, rv.x, y[i][0]);
        y[i][1] = fmaf(xe, rv.y, y[i][1]);
        y[i][2] = fmaf(xe, rv.z, y[i][2]);
        y[i][3] = fmaf(xe, rv.w, y[i][3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (r4 + i < nr)
        *reinterpret_cast<float4*>(X + (r0 + r4 + i) * 64 + c4) =
            make_float4(y[i][0], y[i][1], y[i][2], y[i][3]);
  }
}
}  // namespace

cudaError_t launch_unrotate(float* x0, float* x1, const float* R, long long rows, int d,
                            uint32_t* err, cudaStream_t stream) {
  if (d == 64) {
    static std::atomic<bool> attr64[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr64[dev]) {
      cudaError_t e = cudaFuncSetAttribute(unrotate64_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, kRot64Smem);
      if (e != cudaSuccess) return e;
      attr64[dev] = true;
    }
    const long long tiles = 2 * ((rows + 63) / 64);
    const int grid = static_cast<int>(tiles < 148 * 4 ? tiles : 148 * 4);
    unrotate64_kernel<<<grid, 256, kRot64Smem, stream>>>(x0, x1, R, rows);
    return cudaGetLastError();
  }
  static std::atomic<bool> attr_set[64];   // per device; racing first calls both set it
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(unrotate_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kRotSmem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const long long tiles = 2 * ((rows + 127) / 128);
  const int grid = static_cast<int>(tiles < 148 * 2 ? tiles : 148 * 2);
  unrotate_kernel<<<grid, kRotThreads, kRotSmem, stream>>>(x0, x1, R, rows, err);
  return cudaGetLastError();
}

template cudaError_t launch_bwd<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                    const CUtensorMap&, const CUtensorMap&, const BwdArgs&,
                                    cudaStream_t, cudaEvent_t, cudaEvent_t);
template cudaError_t launch_bwd<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                     const CUtensorMap&, const CUtensorMap&, const BwdArgs&,
                                     cudaStream_t, cudaEvent_t, cudaEvent_t);

}  // namespace fa

#ifdef FA_BWD_TRACE
// Copies the trace stamps of the last traced launch to host memory (3 x 8192 words).
extern "C" __attribute__((visibility("default"))) int fa_bwd_trace_read(void* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, fa::g_bwd_trace, sizeof(fa::g_bwd_trace)));
}
#endif
