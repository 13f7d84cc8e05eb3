// fwd.cu — fused one-pass attention forward for sm_100a (bf16 in, fp32
// accumulate, bf16 O and fp32 logsumexp out).
//
// Algorithm ("FlashAttention系列优化", FlashAttentionV2; "Flash Attention
// 再学习", 1-pass FlashAttention): Q row blocks form the outer loop (one CTA
// owns two 128-row Q tiles), K/V blocks of 128 rows the inner loop. Per row
// the kernel keeps a running max m and running sum l, keeps O unnormalised,
// rescales it by exp(m_old - m_new) when m moves, and divides by l once at the
// end; L = m + log l is the only statistic written (91haoming.cn repost,
// "前向傳播改進").
//
// B200 mapping (the pages' A100/H100 warp layouts are prior art only):
//   warp 0        TMA producer: Q tiles once, then K_j, V_j through an
//                 NSTAGE-deep shared-memory ring guarded by full/empty
//                 mbarriers (the producer/consumer circular buffer of
//                 FlashAttention-3, with TMA).
//   warp 1        allocates TMEM; lane 0 issues every tcgen05.mma:
//                 S_t = Q_t K_j^T (smem x smem -> TMEM fp32) and
//                 O_t += P_t V_j (P from TMEM x V from smem -> TMEM fp32).
//   warps 4..7    softmax for Q tile 0, warps 8..11 for Q tile 1: each
//                 thread owns one row (one TMEM lane), so the row max and row
//                 sum need no shuffles. While one tile's softmax runs, the
//                 tensor core works on the other tile (ping-pong). P goes
//                 out in two halves of 64 keys: P.V starts on the first while
//                 the exps of the second run.
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+D),
// O_1 [256+D, 256+2D). P_t (bf16, packed 2 per column) overwrites the first
// 64 columns of S_t and feeds the P.V MMA directly from TMEM.
// Rescale skipping: m is only moved when a new row max exceeds it by more
// than 2^8 in exp2 units; until then exp2(x - m) <= 256, which fp32 and bf16
// hold exactly as well as values <= 1. The final O / l and L = m + log l use
// the same m, so the result is the same exact quantity.
#include <atomic>

#include "prim.cuh"
#include "kernels.h"

namespace fa {

// Softmax trace (built only with -DFA_FWD_TRACE by exact_attention_102_b200.trace_fwd,
// never in libfa.so): in CTA 0 of the forward, lane 0 of the first softmax warp
// of each tile records clock64 stamps around the steps of every key block.
#ifdef FA_FWD_TRACE
__device__ unsigned long long g_fwd_trace[2][4096];
#define FA_FWD_STAMP(tag)                                                                 \
  do {                                                                                    \
    if (tr_on && tr_n < 4096)                                                             \
      g_fwd_trace[t][tr_n++] = (static_cast<unsigned long long>(clock64()) << 8) | (tag); \
  } while (0)
#else
#define FA_FWD_STAMP(tag) \
  do {                    \
  } while (0)
#endif

namespace {

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;                 // Q rows per tile
  static constexpr int BN = 128;                 // K/V rows per tile
  static constexpr int TILE = 128 * D * 2;       // bytes of one 128-row bf16 tile
  static constexpr int CHUNK = 128 * 128;        // bytes of one 64-column (128 B) chunk
  static constexpr int NCHUNK = D / 64;
  static constexpr int NSTAGE = (D == 128) ? 4 : 8;
  static constexpr int Q_OFF = 0;
  static constexpr int RING_OFF = 2 * TILE;
  static constexpr int BAR_OFF = RING_OFF + NSTAGE * TILE;
  // barriers: q_full | kv_full[NSTAGE] | kv_empty[NSTAGE] | s_full[2] | p_full[2] | o_full[2] | drain
  static constexpr int B_Q = 0;
  static constexpr int B_KVF = 1;
  static constexpr int B_KVE = 1 + NSTAGE;
  static constexpr int B_S = 1 + 2 * NSTAGE;
  static constexpr int B_P = B_S + 2;
  static constexpr int B_O = B_P + 2;
  static constexpr int B_P0 = B_O + 2;          // first 64 keys of P_t in TMEM
  static constexpr int B_DRAIN = B_P0 + 2;
  static constexpr int NBAR = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;  // tmem slot (4 B), abort flag (4 B)
  // block-sparse form: the CTA's key blocks (union of its two tiles' blocks),
  // uint16 ids, uint8 per-tile flags, and three counts
  static constexpr int MAX_UNION = 512;
  static constexpr int UNION_OFF = MISC_OFF + 16;
  static constexpr int SMEM_BYTES = UNION_OFF + 3 * MAX_UNION + 16 + 1024;  // + alignment slack
  // TMEM column of S_t / P_t and of O_t
  static __device__ __forceinline__ uint32_t s_col(int t) { return 128u * t; }
  static __device__ __forceinline__ uint32_t o_col(int t) { return 256u + D * t; }
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr int THREADS = 384;
};

// every kPolyEvery-th pair of scores takes exp2 from exp2_poly_x2 (0: none)
#ifndef FA_FWD_POLY_EVERY
#define FA_FWD_POLY_EVERY 0
#endif
constexpr int kPolyEvery = FA_FWD_POLY_EVERY;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kOrderMax = 256;             // paged form: sequences ordered by context length

// wait-site ids (reported in the device error word)
enum : uint32_t {
  kSiteQ = 1, kSiteKvEmpty = 2, kSiteKvFull = 3, kSiteS = 4, kSiteP = 5,
  kSiteEpi = 7, kSiteDrain = 8
};

// MODE (compile time, so each form carries only its own indexing):
//   kBhnd  [B, H, N, d] tensors;
//   kPacked packed variable-length Q / K / V (FwdArgs.cu_q, cu_k);
//   kPaged  packed Q, keys gathered from a paged cache (FwdArgs.block_table).
//   kSparse [B, H, N, d] tensors with a 128 x 128 block mask (FwdArgs.block_mask).
//   kDropout [B, H, N, d] tensors with dropout on P (FwdArgs.dropout): the
//           P.V operand carries P o Z, the row sums keep the undropped P, and
//           O is scaled by 1 / (keep probability) at the end.
enum { kBhnd = 0, kPacked = 1, kPaged = 2, kSparse = 3, kDropout = 4 };

template <int D, int MODE>
__global__ void __launch_bounds__(384, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, FwdArgs a) {
  using C = FwdCfg<D>;
  // launched with programmatic serialization: the kernel before this one may
  // still be finishing, and anything read below may be its output
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BH = a.B * a.H;
  constexpr bool packed = MODE == kPacked || MODE == kPaged;
  // [B, H, N, d] forms: (batch, head) slices in groups of FwdArgs.head_group,
  // heaviest pair first inside a group, so the running CTAs cover few heads
  // and share their K / V rows in L2 (the host groups only when K and V
  // outgrow L2). Packed forms: heaviest pair first over all (sequence, head)
  // slots.
  int pair, bh;
  if (packed) {
    pair = a.n_pairs - 1 - static_cast<int>(blockIdx.x) / BH;
    bh = static_cast<int>(blockIdx.x) % BH;
  } else {
    const int G = a.head_group > 0 ? min(a.head_group, BH) : BH;
    const int g = static_cast<int>(blockIdx.x) / (G * a.n_pairs);
    const int gsize = min(G, BH - g * G);
    const int r = static_cast<int>(blockIdx.x) - g * G * a.n_pairs;
    pair = a.n_pairs - 1 - r / gsize;
    bh = g * G + r % gsize;
  }

  // The problem this CTA works on: Lq queries against Lk keys. BHND: one
  // (batch, head) slice of length N, TMA coordinates (row, bh). Packed mode:
  // sequence b of the batch, TMA coordinates (head, token).
  constexpr bool paged = MODE == kPaged;
  constexpr bool sparse = MODE == kSparse;
  constexpr bool dropout = MODE == kDropout;
  // P published in two halves (P.V starts on the first 64 keys while the
  // exps of the rest run); the block-sparse form publishes it whole (its
  // skipped blocks and union bookkeeping leave no registers for the split)
  constexpr bool split_p = !sparse;
  int Lq = a.N, Lk = a.N, tq0 = 0, tk0 = 0, hq = 0, hk = 0;
  int seq = 0;                        // packed forms: the sequence of this CTA
  if (packed) {
    // Paged form, longest context first: within each wave of pairs, the CTAs
    // of the sequence with the r-th longest context (ties by index) come r-th,
    // so long contexts do not end up in the tail of the grid (chunks of equal
    // length over contexts of very unequal length). Up to kOrderMax sequences;
    // beyond that, and in the plain packed form, batch order.
    int b = bh / a.H;
    static_assert(3 * C::MAX_UNION + 16 >= 4 * (kOrderMax + 1), "order list exceeds its area");
    if (paged && a.B <= kOrderMax) {
      int* klen = reinterpret_cast<int*>(smem + C::UNION_OFF);   // unused by these forms
      int* pick = klen + kOrderMax;
      for (int s_ = threadIdx.x; s_ < a.B; s_ += blockDim.x)
        klen[s_] = a.ctx[s_];
      if (threadIdx.x == 0) *pick = b;
      __syncthreads();
      for (int s_ = threadIdx.x; s_ < a.B; s_ += blockDim.x) {
        const int ls = klen[s_];
        int r = 0;
        for (int u = 0; u < a.B; ++u) r += klen[u] > ls || (klen[u] == ls && u < s_);
        if (r == b) *pick = s_;
      }
      __syncthreads();
      b = *pick;
    }
    seq = b;
    hq = bh % a.H;
    hk = hq / (a.H / a.Hkv);
    tq0 = a.cu_q[b];
    Lq = a.cu_q[b + 1] - tq0;
    if (paged) {                      // paged keys: the sequence's cached tokens
      Lk = a.ctx[b];
    } else {
      tk0 = a.cu_k[b];
      Lk = a.cu_k[b + 1] - tk0;
    }
    const long long k_end = paged ? static_cast<long long>(a.max_blocks) * 16
                                                     : static_cast<long long>(a.Tk) - tk0;
    if (tq0 < 0 || tk0 < 0 || Lq < 0 || Lk < 0 || Lq > a.N || tq0 + Lq > a.Tq || Lk > k_end) {
      if (threadIdx.x == 0 && pair == a.n_pairs - 1) atomicCAS(a.err, 0u, kErrBadIndex + 1);
      Lq = 0;                       // nothing is read or written for this sequence
      Lk = 0;
    }
  }
  // causal: query row i sees keys j <= i + off (off = 0 when Lq == Lk)
  const int off = a.causal ? Lk - Lq : 0;
  const int nkb = (Lk + C::BN - 1) / C::BN;

  // per-tile extent: rows [q0, q0+128), key blocks [0, nkb_t); a tile with rows
  // but no visible key (nkb_t = 0) still writes O = 0 and L = -inf
  int q0[2], nkb_t[2];
  bool rows_t[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    q0[t] = (pair * 2 + t) * C::BM;
    rows_t[t] = q0[t] < Lq;
    const int last_key = min(q0[t] + C::BM - 1, Lq - 1) + off;  // causal: last key any row sees
    nkb_t[t] = !rows_t[t] ? 0 : !a.causal ? nkb : last_key < 0 ? 0 : min(nkb, last_key / C::BN + 1);
  }
  int nkb_cta = max(nkb_t[0], nkb_t[1]);
  // Block-sparse form: the CTA walks the union of its two tiles' active key
  // blocks; a tile takes part in the first cnt_t union steps (those below its
  // causal limit) and treats a step whose block it does not see as fully masked.
  uint16_t* ulist = reinterpret_cast<uint16_t*>(smem + C::UNION_OFF);
  uint8_t* uflag = smem + C::UNION_OFF + 2 * C::MAX_UNION;
  int* ucount = reinterpret_cast<int*>(smem + C::UNION_OFF + 3 * C::MAX_UNION);
  if constexpr (sparse) {
    if (threadIdx.x == 0) {
      const int nkb_all = (a.N + C::BN - 1) / C::BN;
      const uint8_t* m0 = a.block_mask + bh * a.mask_bh_stride + static_cast<long long>(2 * pair) * nkb_all;
      const uint8_t* m1 = m0 + nkb_all;
      int n = 0, c0 = 0, c1 = 0;
      for (int j = 0; j < nkb_cta && n < C::MAX_UNION; ++j) {
        const bool a0 = j < nkb_t[0] && m0[j] != 0;
        const bool a1 = j < nkb_t[1] && m1[j] != 0;
        if (!(a0 || a1)) continue;
        ulist[n] = static_cast<uint16_t>(j);
        uflag[n] = static_cast<uint8_t>((a0 ? 1 : 0) | (a1 ? 2 : 0));
        ++n;
        if (j < nkb_t[0]) c0 = n;
        if (j < nkb_t[1]) c1 = n;
      }
      ucount[0] = c0;
      ucount[1] = c1;
      ucount[2] = n;
    }
  }
  // TMA coordinates (y, z) of Q row q and of K / V row k of this problem
  auto q_yz = [&](int q) { return packed ? make_int2(hq, tq0 + q) : make_int2(q, bh); };
  auto k_yz = [&](int k) { return packed ? make_int2(hk, tk0 + k) : make_int2(k, bh); };

  auto bar = [&](int i) -> uint32_t { return base + C::BAR_OFF + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_Q), 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar(C::B_KVF + s), 1);
      mbar_init(bar(C::B_KVE + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C::B_S + t), 1);
      mbar_init(bar(C::B_P + t), 4);   // one arrival per softmax warp
      mbar_init(bar(C::B_O + t), 1);
      mbar_init(bar(C::B_P0 + t), 4);
    }
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
  if constexpr (sparse) {                         // union steps replace key blocks
    nkb_t[0] = ucount[0];
    nkb_t[1] = ucount[1];
    nkb_cta = ucount[2];
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int nq = (nkb_t[0] > 0) + (nkb_t[1] > 0);
      mbar_arrive_expect_tx(bar(C::B_Q), nq * C::TILE);
      for (int t = 0; t < 2; ++t) {
        if (nkb_t[t] == 0) continue;
        const int2 yz = q_yz(q0[t]);
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_3d(base + C::Q_OFF + t * C::TILE + c * C::CHUNK, &tmQ, bar(C::B_Q), c * 64,
                      yz.x, yz.y);
      }
      int it = 0;
      bool ok = true;
      for (int j = 0; j < nkb_cta && ok; ++j) {
        // paged keys: the 8 physical 16-token blocks of key block j (a block
        // past the context reads block 0, masked like a tail; an id outside the
        // pool is recorded and replaced by 0)
        int phys[C::BN / 16];
        if (paged) {
#pragma unroll
          for (int t = 0; t < C::BN / 16; ++t) {
            const int lb = j * (C::BN / 16) + t;
            int pb = lb * 16 < Lk ? a.block_table[static_cast<size_t>(seq) * a.max_blocks + lb] : 0;
            if (pb < 0 || pb >= a.num_phys) {
              atomicCAS(a.err, 0u, kErrBadIndex + 4);
              pb = 0;
            }
            phys[t] = (pb * a.Hkv + hk) * 16;
          }
        }
        for (int w = 0; w < 2 && ok; ++w, ++it) {
          const int s = it % C::NSTAGE;
          const uint32_t ph = (it / C::NSTAGE) & 1;
          ok = mbar_wait(bar(C::B_KVE + s), ph ^ 1, a.err, kSiteKvEmpty, abort_flag);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(C::B_KVF + s), C::TILE);
          const CUtensorMap* m = (w == 0) ? &tmK : &tmV;
          if (paged) {
            // eight 16-row boxes, each at its own row of the swizzled tile
            for (int t = 0; t < C::BN / 16; ++t)
              for (int c = 0; c < C::NCHUNK; ++c)
                tma_load_3d(base + C::RING_OFF + s * C::TILE + c * C::CHUNK + t * 16 * 128, m,
                            bar(C::B_KVF + s), c * 64, phys[t], 0);
          } else {
            const int2 yz = k_yz((sparse ? ulist[j] : j) * C::BN);
            for (int c = 0; c < C::NCHUNK; ++c)
              tma_load_3d(base + C::RING_OFF + s * C::TILE + c * C::CHUNK, m, bar(C::B_KVF + s),
                          c * 64, yz.x, yz.y);
          }
        }
      }
      // drain: make sure the last loads issued have landed before teardown
      const int issued = it;
      for (int k = max(0, issued - C::NSTAGE); k < issued; ++k)
        mbar_wait(bar(C::B_KVF + k % C::NSTAGE), (k / C::NSTAGE) & 1, a.err, kSiteDrain,
                  nullptr, 200000000ull);
      if (nq) mbar_wait(bar(C::B_Q), 0, a.err, kSiteDrain, nullptr, 200000000ull);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idS = idesc_f16(128, C::BN, 1, 0, 0);
      constexpr uint32_t idPV = idesc_f16(128, D, 1, 0, 1);
      // Issue order per key block j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1).
      // tcgen05.mma from one thread executes in issue order, so S_t(j+1) may
      // overwrite the P_t(j) columns PV_t(j) reads without waiting for it;
      // the commit after S_t(j+1) also tells the softmax that PV_t(j) is done
      // (its O rescale for block j+1 relies on that).
      int it = 0;
      int npv[2] = {0, 0};
      bool ok = mbar_wait(bar(C::B_Q), 0, a.err, kSiteQ, abort_flag);
      // descriptors of Q tile 0 and ring stage 0; a tile at a byte offset is the
      // base descriptor plus offset / 16 (start-address field)
      const uint64_t dQ = smem_desc_sw128(base + C::Q_OFF, 16, 1024);        // K-major
      const uint64_t dK = smem_desc_sw128(base + C::RING_OFF, 16, 1024);     // K-major
      const uint64_t dVm = smem_desc_sw128(base + C::RING_OFF, C::CHUNK, 1024);  // MN-major
      auto add = [](uint64_t d, uint32_t bytes) -> uint64_t { return d + (bytes >> 4); };
      auto issue_s = [&](int t, int stage) {
        const uint64_t q = add(dQ, t * C::TILE), k = add(dK, stage * C::TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::CHUNK + (kk & 3) * 32;
          umma_f16_ss(tmem + C::s_col(t), add(q, off), add(k, off), idS, kk > 0);
        }
        umma_commit(bar(C::B_S + t));
      };
      if (ok && nkb_cta > 0) {        // K_0
        const int s = it % C::NSTAGE;
        ok = mbar_wait(bar(C::B_KVF + s), (it / C::NSTAGE) & 1, a.err, kSiteKvFull, abort_flag);
        ++it;
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (nkb_t[t] > 0) issue_s(t, s);
          umma_commit(bar(C::B_KVE + s));
        }
      }
      for (int j = 0; j < nkb_cta && ok; ++j) {
        const int sv = it % C::NSTAGE;  // V_j
        ok = mbar_wait(bar(C::B_KVF + sv), (it / C::NSTAGE) & 1, a.err, kSiteKvFull, abort_flag);
        if (!ok) break;
        ++it;
        const uint64_t vm = add(dVm, sv * C::TILE);
        int sk = -1;                    // ring stage of K_{j+1}, once waited for
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= nkb_t[t]) continue;
          // P.V(j) in two halves of 64 keys, each as soon as its half of P is in
          // (the block-sparse form: all of P at once)
          if constexpr (split_p) {
            ok = mbar_wait(bar(C::B_P0 + t), npv[t] & 1, a.err, kSiteP, abort_flag);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < C::BN / 32; ++kk)
              umma_f16_ts(tmem + C::o_col(t), tmem + C::s_col(t) + kk * 8, add(vm, kk * 2048),
                          idPV, (npv[t] > 0 || kk > 0) ? 1u : 0u);
          }
          ok = mbar_wait(bar(C::B_P + t), npv[t] & 1, a.err, kSiteP, abort_flag);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = split_p ? C::BN / 32 : 0; kk < C::BN / 16; ++kk)
            umma_f16_ts(tmem + C::o_col(t), tmem + C::s_col(t) + kk * 8, add(vm, kk * 2048), idPV,
                        (npv[t] > 0 || kk > 0) ? 1u : 0u);
          if (j + 1 == nkb_t[t]) umma_commit(bar(C::B_O + t));   // last P.V of tile t
          ++npv[t];
          if (j + 1 < nkb_t[t]) {
            if (sk < 0) {
              sk = it % C::NSTAGE;
              ok = mbar_wait(bar(C::B_KVF + sk), (it / C::NSTAGE) & 1, a.err, kSiteKvFull,
                             abort_flag);
              ++it;
              if (!ok) break;
              tc_fence_after();
            }
            issue_s(t, sk);
          }
        }
        if (!ok) break;
        umma_commit(bar(C::B_KVE + sv));             // V_j: both PV_t(j) issued before
        if (sk >= 0) umma_commit(bar(C::B_KVE + sk));  // K_{j+1}: both S_t(j+1) issued before
      }
      // drain every MMA this thread issued before TMEM is released
      umma_commit(bar(C::B_DRAIN));
      mbar_wait(bar(C::B_DRAIN), 0, a.err, kSiteDrain, nullptr, 200000000ull);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int t = (warp - 4) >> 2;
    const int r = (warp & 3) * 32 + lane;           // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + C::s_col(t);
    const uint32_t o_addr = tmem + lane_off + C::o_col(t);
    const int row = q0[t] + r;
    const int limit = a.causal ? min(row + off, Lk - 1) : Lk - 1;  // last visible key (< 0: none)
    const float sl2 = a.scale_log2;
    float m_run = -INFINITY;
    float l_run = 0.f;    // sum of fp32 P
    float lr_run = 0.f;   // sum of bf16-rounded P
    bool ok = true;
#ifdef FA_FWD_TRACE
    const bool tr_on = blockIdx.x == 0 && lane == 0 && (warp & 3) == 0;
    int tr_n = 0;
#endif
    for (int j = 0; j < nkb_t[t]; ++j) {
      FA_FWD_STAMP(1);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::B_S + t), j & 1, a.err, kSiteS, abort_flag));
      if (!ok) break;
      FA_FWD_STAMP(2);
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(s_addr + c * 32, sr[c]);
      tmem_ld_wait();
      FA_FWD_STAMP(3);
#define SV(c) __uint_as_float(sr[(c) >> 5][(c)&31])
      if (sparse && !((uflag[j] >> t) & 1)) {   // a block this tile does not see: P = 0
        uint32_t zero[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) zero[c] = 0u;
        tmem_st32(s_addr, zero);
        tmem_st32(s_addr + 32, zero);
        tmem_st_wait();
        tc_fence_before();
        warp_arrive(bar(C::B_P + t));
        continue;
      }
      const int kbase = (sparse ? ulist[j] : j) * C::BN;
      if (kbase + C::BN - 1 > limit) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (kbase + c > limit) sr[c >> 5][c & 31] = 0xff800000u;  // -inf
      }
      float mx0 = SV(0), mx1 = SV(1), mx2 = SV(2), mx3 = SV(3);
#pragma unroll
      for (int c = 4; c < 124; c += 8) {
        mx0 = fmax3(mx0, SV(c), SV(c + 1));
        mx1 = fmax3(mx1, SV(c + 2), SV(c + 3));
        mx2 = fmax3(mx2, SV(c + 4), SV(c + 5));
        mx3 = fmax3(mx3, SV(c + 6), SV(c + 7));
      }
      mx0 = fmax3(mx0, SV(124), SV(125));
      mx1 = fmax3(mx1, SV(126), SV(127));
      const float mx = fmax3(fmax3(mx0, mx1, mx2), mx3, mx3) * sl2;
      float alpha = 1.f;
      if (mx > m_run + kRescaleThreshold) {  // also true for the first block (m_run = -inf)
        alpha = ex2_approx(m_run - mx);      // exp2(-inf) = 0 on the first block
        m_run = mx;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      // Two row sums: l_run of the fp32 probabilities (for L = m + log l) and
      // lr_run of the bf16-rounded P the P.V product consumes (for O = acc/l),
      // so the normalisation weighs every key exactly as the numerator does.
      // pairs of scores on packed fp32; every kPolyEvery-th pair takes its
      // exp2 from the polynomial, the rest from the special-function unit
      const uint64_t sl2x2 = f2_pack(sl2, sl2), negm2 = f2_pack(-m_use, -m_use);
      uint64_t la = 0, lb = 0, ra = 0, rb = 0;     // (0.f, 0.f) pairs
      uint4 rnd = make_uint4(0u, 0u, 0u, 0u);     // dropout: random bytes of 16 keys
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        uint32_t pk[32];
#pragma unroll
        for (int qq = 0; qq < 32; ++qq) {
          const int q = 32 * hq + qq;
          if (dropout && (q & 7) == 0)
            rnd = philox4x32_10(static_cast<uint32_t>((kbase >> 4) + (q >> 3)),
                                static_cast<uint32_t>(row), static_cast<uint32_t>(bh),
                                a.drop_offset, a.seed_lo, a.seed_hi);
          const uint64_t x2 = f2_fma(f2_pack(SV(2 * q), SV(2 * q + 1)), sl2x2, negm2);
          uint64_t p2;
          if (kPolyEvery > 0 && q % (kPolyEvery > 0 ? kPolyEvery : 1) == kPolyEvery - 1) {
            p2 = exp2_poly_x2(x2);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
          }
          float p0, p1;
          f2_unpack(p2, p0, p1);
          const uint32_t u = pack_bf16x2(p0, p1);
          const uint64_t rr = f2_pack(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
          if (q & 1) {
            lb = f2_add(lb, p2);
            rb = f2_add(rb, rr);
          } else {
            la = f2_add(la, p2);
            ra = f2_add(ra, rr);
          }
          uint32_t us = u;                           // P, or P o Z under dropout
          if (dropout) {
            const int wi = (q & 7) >> 1;             // keys 2q, 2q+1: bytes 2(q&1), +1 of word wi
            const uint32_t w = wi == 0 ? rnd.x : wi == 1 ? rnd.y : wi == 2 ? rnd.z : rnd.w;
            us &= (q & 1) ? keep_halves<1>(w, a.drop_bias) : keep_halves<0>(w, a.drop_bias);
          }
          pk[qq] = us;
        }
        tmem_st32(s_addr + 32 * hq, pk);
        if (split_p && hq == 0) {
          // O rescale before P.V(j) starts on the first 64 keys (PV of block
          // j-1 has completed: S_t(j)'s commit covers it)
          if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
            FA_FWD_STAMP(9);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t orr[32];
              tmem_ld32(o_addr + c * 32, orr);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e)
                orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
              tmem_st32(o_addr + c * 32, orr);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          warp_arrive(bar(C::B_P0 + t));                 // the first 64 keys: P.V may start
          FA_FWD_STAMP(4);
        }
      }
      FA_FWD_STAMP(5);
      if constexpr (!split_p) {
        // O rescale (PV of block j-1 has completed: S_t(j)'s commit covers it)
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          FA_FWD_STAMP(9);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            tmem_ld32(o_addr + c * 32, orr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e)
              orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
            tmem_st32(o_addr + c * 32, orr);
          }
        }
      }
#undef SV
      float l0, l1, l2, l3, r0, r1, r2, r3;
      f2_unpack(la, l0, l1);
      f2_unpack(lb, l2, l3);
      f2_unpack(ra, r0, r1);
      f2_unpack(rb, r2, r3);
      l_run = l_run * alpha + ((l0 + l1) + (l2 + l3));
      lr_run = lr_run * alpha + ((r0 + r1) + (r2 + r3));
      tmem_st_wait();
      FA_FWD_STAMP(6);
      tc_fence_before();
      warp_arrive(bar(C::B_P + t));
      FA_FWD_STAMP(7);
    }
    // ------------------------------------------------------------ epilogue
    // output row of query `row`: BHND [bh][row] or packed [token][head]
    const size_t orow_idx = packed ? static_cast<size_t>(tq0 + row) * a.H + hq
                                   : static_cast<size_t>(bh) * a.N + row;
    const size_t lse_idx = packed ? static_cast<size_t>(hq) * a.Tq + tq0 + row
                                  : static_cast<size_t>(bh) * a.N + row;
    if (ok && nkb_t[t] == 0 && rows_t[t] && row < Lq) {   // sees no key: O = 0, L = -inf
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.o) + orow_idx * D);
#pragma unroll
      for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
      a.lse[lse_idx] = -INFINITY;
    }
    if (ok && nkb_t[t] > 0) {
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bar(C::B_O + t), 0, a.err, kSiteEpi, abort_flag));
      if (ok) {
        tc_fence_after();
        // a row that saw no key has l = 0: O = 0, and L = m + log l = -inf
        const float inv_l = lr_run > 0.f ? (dropout ? a.drop_scale : 1.f) / lr_run : 0.f;
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + orow_idx * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(o_addr + c * 32, orr);
          tmem_ld_wait();
          if (row < Lq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int b = 8 * e;
              dst[e] = make_uint4(
                  pack_bf16x2(__uint_as_float(orr[b + 0]) * inv_l, __uint_as_float(orr[b + 1]) * inv_l),
                  pack_bf16x2(__uint_as_float(orr[b + 2]) * inv_l, __uint_as_float(orr[b + 3]) * inv_l),
                  pack_bf16x2(__uint_as_float(orr[b + 4]) * inv_l, __uint_as_float(orr[b + 5]) * inv_l),
                  pack_bf16x2(__uint_as_float(orr[b + 6]) * inv_l, __uint_as_float(orr[b + 7]) * inv_l));
            }
          }
        }
        if (row < Lq) a.lse[lse_idx] = (m_run + log2f(l_run)) * 0.6931471805599453f;
      }
    }
    tc_fence_before();
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
int fwd_smem_bytes() {
  return FwdCfg<D>::SMEM_BYTES;
}

template <int D>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdArgs& a, cudaStream_t stream) {
  using C = FwdCfg<D>;
  static std::atomic<bool> attr_set[64];   // per device; racing first calls both set it
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    for (auto fn : {fwd_kernel<D, kBhnd>, fwd_kernel<D, kPacked>, fwd_kernel<D, kPaged>,
                    fwd_kernel<D, kSparse>, fwd_kernel<D, kDropout>}) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           C::SMEM_BYTES);
      if (e != cudaSuccess) return e;
    }
    attr_set[dev] = true;
  }
  const int grid = a.n_pairs * a.B * a.H;
  void (*k)(CUtensorMap, CUtensorMap, CUtensorMap, FwdArgs) =
      a.dropout ? fwd_kernel<D, kDropout>
      : a.block_mask != nullptr ? fwd_kernel<D, kSparse>
      : a.block_table != nullptr ? fwd_kernel<D, kPaged>
      : a.cu_q != nullptr ? fwd_kernel<D, kPacked> : fwd_kernel<D, kBhnd>;
  cudaError_t e = launch_pdl(k, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, stream, tq, tk, tv, a);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

template cudaError_t launch_fwd<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                    const FwdArgs&, cudaStream_t);
template cudaError_t launch_fwd<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                     const FwdArgs&, cudaStream_t);

}  // namespace fa

#ifdef FA_FWD_TRACE
// Copies the trace stamps of the last traced launch to host memory (2 x 4096 words).
extern "C" __attribute__((visibility("default"))) int fa_fwd_trace_read(void* host) {
  return static_cast<int>(cudaMemcpyFromSymbol(host, fa::g_fwd_trace, sizeof(fa::g_fwd_trace)));
}
#endif
