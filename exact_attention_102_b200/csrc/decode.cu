// decode.cu — single-token attention over a paged KV cache (memory bound).
//
// "FlashAttention系列优化" (johneyzheng.top), section PagedAttention: the KV
// cache of a sequence lives in fixed-size physical blocks reached through a
// per-sequence block table; several sequences (parallel sampling) may point
// at the same physical block. The kernel only follows the table.
//
// Work split: one work item per (sequence, KV head, split of `split_blocks`
// 16-token blocks); a persistent grid of two CTAs per SM takes items from a
// global counter. An item serves the G = Hq / Hkv (1 .. 8) query heads that
// share its KV head, so every K/V byte is read from HBM once per query group.
// Head dimension d = 64 or 128 (a template parameter). Each split produces a
// partial (O_s normalised over its own keys, L_s = its logsumexp); the
// combine kernel merges the splits with L = log sum_s exp(L_s),
// O = sum_s exp(L_s - L) O_s, which follows from the definition of the
// logsumexp statistic (91haoming.cn repost, "前向傳播改進").
//
// Inside a CTA:
//   warp 4 (producer)  per item: the split's slice of the block table and the
//                      G query heads (one bulk copy); then, per table entry,
//                      the (block, KV head) K and V slabs (16 tokens x d bf16)
//                      as d / 64 TMA boxes of 64 columns each, 128-byte
//                      swizzled, into an 8-stage ring (full / empty mbarriers).
//   warps 0..3         warp w takes blocks w, w+4, ... of the item and keeps its
//                      own online-softmax state. Per block: S = Q K^T and
//                      O += P V on the tensor cores with mma.sync m16n8k16
//                      (bf16 in, fp32 accumulate; the G query heads fill G of
//                      the 16 rows), K and V fragments read with ldmatrix from
//                      the swizzled tiles; the S accumulator fragment is the P
//                      operand fragment of the P.V product, so P never leaves
//                      registers. The four warp states are merged at the end of
//                      the item with the logsumexp rule.
// Scores per block are a few thousand multiply-adds against 8 KB of HBM
// traffic; the tensor cores only remove instruction-issue pressure so the
// kernel can keep HBM busy.
#include <atomic>

#include "prim.cuh"
#include "kernels.h"

namespace fa {

namespace {

constexpr int kBlk = 16;          // tokens per physical block
constexpr int kMaxGroup = 8;      // query heads per KV head: 1 .. 8 (rows of the m16 MMA)
constexpr int kStages = 8;
constexpr int kMaxSplitBlocks = 128;
constexpr int kComputeWarps = 4;
constexpr int kComputeThreads = 32 * kComputeWarps;
constexpr int kThreads = kComputeThreads + 32;
constexpr float kRescaleThreshold = 8.0f;

// Shared memory layout (bytes) for head dimension D; the ring is 1024-byte
// aligned for the 128-byte swizzle. A (block, KV head) K or V slab is 16
// tokens x D bf16, brought in as D / 64 TMA boxes of 64 columns (2 KB each).
template <int D>
struct DecCfg {
  static constexpr int kSlab = kBlk * D * 2;
  static constexpr int kBox = kBlk * 128;
  static constexpr int kStageBytes = 2 * kSlab;                     // K + V
  static constexpr int kRingOff = 0;
  static constexpr int kMergeOff = kRingOff + kStages * kStageBytes;  // [4 warps][8 heads][D] fp32
  static constexpr int kQOff = kMergeOff + kComputeWarps * kMaxGroup * D * 4;
  static constexpr int kQBytes = kMaxGroup * D * 2;                 // one q group buffer
  static constexpr int kTableOff = kQOff + 2 * kQBytes;
  static constexpr int kDescOff = kTableOff + 2 * kMaxSplitBlocks * 4;  // 2 x {seq, kvh, split, nb, rem}
  static constexpr int kBarOff = kDescOff + 2 * 32;   // full[S] empty[S] qfull[2] qempty[2] merge
  static constexpr int kRedOff = kBarOff + (2 * kStages + 5) * 8;  // m, l: [4 warps][8 heads] x 2
  static constexpr int kMiscOff = kRedOff + 2 * kComputeWarps * kMaxGroup * 4;
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
};

enum : uint32_t {
  kSiteFull = 0x21, kSiteEmpty = 0x22, kSiteDrain = 0x23, kSiteQ = 0x24, kSiteMerge = 0x25
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D(16x8 fp32) += A(16x16 bf16, row) * B(16x8 bf16, col)
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Persistent split kernel (see the file comment). Shared tiles: each 64-column
// box of a slab is [16 rows][128 B], 16-byte units XOR-swizzled with
// (row % 8) by the TMA.
template <int D>
__global__ void __launch_bounds__(kThreads, 2)
decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    DecodeArgs a) {
  using C = DecCfg<D>;
  constexpr int kSlab = C::kSlab, kBox = C::kBox, kStageBytes = C::kStageBytes;
  constexpr int NB = D / 64;            // TMA boxes per slab
  constexpr int KS = D / 16;            // k-steps of S = Q K^T
  constexpr int NT = D / 8;             // n-tiles of O = P V
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw_addr);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int G = a.group;
  int* table = reinterpret_cast<int*>(smem + C::kTableOff);
  int* desc = reinterpret_cast<int*>(smem + C::kDescOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff);
  auto full = [&](int s) -> uint32_t { return sbase + C::kBarOff + 8 * s; };
  auto empty = [&](int s) -> uint32_t { return sbase + C::kBarOff + 8 * (kStages + s); };
  auto qfull = [&](int p) -> uint32_t { return sbase + C::kBarOff + 8 * (2 * kStages + p); };
  auto qempty = [&](int p) -> uint32_t { return sbase + C::kBarOff + 8 * (2 * kStages + 2 + p); };
  const uint32_t merge_bar = sbase + C::kBarOff + 8 * (2 * kStages + 4);
  const long long total = static_cast<long long>(a.max_splits) * a.Hkv * a.num_seqs;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);                    // one consumer warp per block
    }
    for (int p = 0; p < 2; ++p) {
      mbar_init(qfull(p), 1);
      mbar_init(qempty(p), kComputeWarps);
    }
    mbar_init(merge_bar, kComputeThreads);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kComputeWarps) {
    // ------------------------------------------------------------ producer
    // Items are handed out dynamically: lane 0 takes the next index of the
    // dense (split, KV head, sequence) space from a global counter and skips
    // splits past a sequence's end. The next item is resolved while the
    // current item's first blocks are in flight.
    struct Item { int seq, kvh, split, nb, rem; };
    auto resolve = [&]() -> Item {     // lane 0 only
      Item it{0, 0, 0, 0, 0};
      while (true) {
        const long long idx = atomicAdd(a.counter, 1u);
        if (idx >= total) return it;   // nb = 0: no more work
        // split-major order: the same split of every (KV head, sequence) runs
        // at about the same time, so blocks that several sequences share
        // (parallel-sampling prefixes, adjacent sequences) are read from HBM
        // once and from L2 for the others
        it.seq = static_cast<int>(idx % a.num_seqs);
        const long long rest = idx / a.num_seqs;
        it.kvh = static_cast<int>(rest % a.Hkv);
        it.split = static_cast<int>(rest / a.Hkv);
        // a length outside [1, max_ctx] is reported by the combine kernel;
        // the clamp keeps the reads inside the table and the workspace
        const int ctx = max(1, min(a.context_lens[it.seq], a.max_ctx));
        const int first = it.split * a.split_blocks;
        const int nblk = (ctx + kBlk - 1) / kBlk;
        if (first < nblk) {
          it.nb = min(nblk - first, a.split_blocks);
          it.rem = min(ctx - first * kBlk, it.nb * kBlk);
          return it;
        }
      }
    };
    auto bcast = [&](Item it) -> Item {
      it.seq = __shfl_sync(0xffffffffu, it.seq, 0);
      it.kvh = __shfl_sync(0xffffffffu, it.kvh, 0);
      it.split = __shfl_sync(0xffffffffu, it.split, 0);
      it.nb = __shfl_sync(0xffffffffu, it.nb, 0);
      it.rem = __shfl_sync(0xffffffffu, it.rem, 0);
      return it;
    };
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    Item cur{0, 0, 0, 0, 0};
    if (lane == 0) cur = resolve();
    cur = bcast(cur);
    long long g = 0;      // blocks issued so far (ring position)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int p = k & 1;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(qempty(p), ((k >> 1) & 1) ^ 1, a.err, kSiteQ, abort_flag));
      if (!ok) break;
      if (cur.nb == 0) {               // no more work: publish the end marker
        if (lane == 0) {
          desc[8 * p + 3] = 0;
          mbar_arrive(qfull(p));
        }
        break;
      }
      int* tab = table + p * kMaxSplitBlocks;
      const int* trow =
          a.block_table + static_cast<size_t>(cur.seq) * a.max_blocks + cur.split * a.split_blocks;
      for (int i = lane; i < cur.nb; i += 32) {
        int id = trow[i];
        if (id < 0 || id >= a.num_phys) {  // never dereference a bad id
          atomicCAS(a.err, 0u, kErrBadIndex + 1);
          id = 0;
        }
        tab[i] = id;
      }
      __syncwarp();
      Item nxt{0, 0, 0, 0, 0};
      if (lane == 0) {
        desc[8 * p + 0] = cur.seq;
        desc[8 * p + 1] = cur.kvh;
        desc[8 * p + 2] = cur.split;
        desc[8 * p + 3] = cur.nb;
        desc[8 * p + 4] = cur.rem;
        const uint32_t qbytes = static_cast<uint32_t>(G) * D * 2;   // G query heads, contiguous
        mbar_arrive_expect_tx(qfull(p), qbytes);
        bulk_load(sbase + C::kQOff + p * C::kQBytes,
                  static_cast<const __nv_bfloat16*>(a.q) +
                      (static_cast<size_t>(cur.seq) * a.Hq + cur.kvh * G) * D,
                  qbytes, qfull(p));
        const int head = min(cur.nb, kStages);
        for (int i = 0; i < cur.nb && ok; ++i, ++g) {
          if (i == head) nxt = resolve();   // overlaps with the blocks in flight
          const int s = static_cast<int>(g % kStages);
          ok = mbar_wait(empty(s), static_cast<uint32_t>((g / kStages) & 1) ^ 1, a.err, kSiteEmpty,
                         abort_flag);
          if (!ok) break;
          const int row = (tab[i] * a.Hkv + cur.kvh) * kBlk;
          const uint32_t st = sbase + C::kRingOff + s * kStageBytes;
          mbar_arrive_expect_tx(full(s), kStageBytes);
#pragma unroll
          for (int c = 0; c < NB; ++c) {
            tma_load_3d(st + c * kBox, &tmK, full(s), 64 * c, row, 0);
            tma_load_3d(st + kSlab + c * kBox, &tmV, full(s), 64 * c, row, 0);
          }
        }
        if (ok && cur.nb <= head) nxt = resolve();
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      cur = bcast(nxt);
    }
    if (lane == 0) {
      for (long long i = (g > kStages ? g - kStages : 0); i < g; ++i)
        mbar_wait(full(static_cast<int>(i % kStages)), static_cast<uint32_t>((i / kStages) & 1),
                  a.err, kSiteDrain, nullptr, 200000000ull);
    }
    return;
  }

  // -------------------------------------------------------------- compute
  // mma.sync fragment coordinates: group g = lane / 4 (A/C row, B column),
  // quad index q = lane % 4 (A/B k pair 2q, 2q+1; C column pair 2q, 2q+1).
  const int g = lane >> 2;
  const int qd = lane & 3;
  const bool real = g < G;              // A/C rows 0..G-1 are the query heads, the rest padding
  float* red = reinterpret_cast<float*>(smem + C::kRedOff);
  float* mrg = reinterpret_cast<float*>(smem + C::kMergeOff);
  uint32_t merge_phase = 0;
  auto sync128 = [&]() -> bool {        // bounded, never bar.sync (see below)
    mbar_arrive(merge_bar);
    const bool r = mbar_wait(merge_bar, merge_phase & 1, a.err, kSiteMerge, abort_flag);
    ++merge_phase;
    return __all_sync(0xffffffffu, r);
  };
  // ldmatrix row addresses inside a stage (bytes from the stage base):
  //  K (non-transposed, B operand of S = Q K^T): matrix mi = lane/8 covers tokens
  //    8*(mi/2) .. +7 and 16-byte unit (mi%2) of the k-step's 32-byte slice.
  //  V (transposed, B operand of O = P V): matrix mi covers tokens 8*(mi%2) .. +7
  //    and the 8 columns of n-tile 2*j + mi/2.
  const int mi = lane >> 3, rr = lane & 7;
  const int k_tok = (mi >> 1) * 8 + rr;
  const int v_tok = (mi & 1) * 8 + rr;
  long long gb = 0;                      // blocks consumed by this CTA (ring position)
  for (int k = 0;; ++k) {
    const int p = k & 1;
    if (!__all_sync(0xffffffffu, mbar_wait(qfull(p), (k >> 1) & 1, a.err, kSiteQ, abort_flag)))
      break;
    const int seq = desc[8 * p + 0], kvh = desc[8 * p + 1], split = desc[8 * p + 2];
    const int nb = desc[8 * p + 3], rem = desc[8 * p + 4];
    if (nb == 0) break;
    // Q fragments (A of S = Q K^T): a0 = Q[g][16ks + 2q, +1], a2 = Q[g][16ks + 8 + 2q, +1]
    uint32_t qa[KS][2];
    {
      const uint32_t* qs = reinterpret_cast<const uint32_t*>(smem + C::kQOff + p * C::kQBytes);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        qa[ks][0] = real ? qs[(g * D + 16 * ks + 2 * qd) >> 1] : 0u;
        qa[ks][1] = real ? qs[(g * D + 16 * ks + 8 + 2 * qd) >> 1] : 0u;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(qempty(p));
    float o[NT][4];                     // O rows g (head) / g+8 (padding), columns 8n + 2q, +1
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;   // per head (quad-uniform m, per-thread partial l)
    bool ok = true;
    for (int i = warp; i < nb; i += kComputeWarps) {
      const long long gi = gb + i;
      const int s = static_cast<int>(gi % kStages);
      ok = __all_sync(0xffffffffu, mbar_wait(full(s), static_cast<uint32_t>((gi / kStages) & 1),
                                             a.err, kSiteFull, abort_flag));
      if (!ok) break;
      const uint32_t st = sbase + C::kRingOff + s * kStageBytes;
      // ---- S (heads x 16 tokens) = Q K^T, two n-tiles of 8 tokens
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int unit = 2 * (ks & 3) + (mi & 1);
        const uint32_t addr = st + (ks >> 2) * kBox + k_tok * 128 + ((unit ^ (k_tok & 7)) << 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(addr, b0, b1, b2, b3);
        mma_bf16(sc[0], qa[ks][0], 0u, qa[ks][1], 0u, b0, b1);
        mma_bf16(sc[1], qa[ks][0], 0u, qa[ks][1], 0u, b2, b3);
      }
      // ---- online softmax over the block's tokens (exp2 units)
      float x[4];
      const int tok0 = i * kBlk + 2 * qd;
      x[0] = (tok0 < rem) ? sc[0][0] * a.scale_log2 : -INFINITY;
      x[1] = (tok0 + 1 < rem) ? sc[0][1] * a.scale_log2 : -INFINITY;
      x[2] = (tok0 + 8 < rem) ? sc[1][0] * a.scale_log2 : -INFINITY;
      x[3] = (tok0 + 9 < rem) ? sc[1][1] * a.scale_log2 : -INFINITY;
      float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      if (mx > m_run + kRescaleThreshold) {   // quad-uniform
        const float alpha = ex2_approx(m_run - mx);  // 0 while m_run = -inf
        m_run = mx;
        l_run *= alpha;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          o[n][0] *= alpha;
          o[n][1] *= alpha;
        }
      }
      const float mu = (m_run == -INFINITY) ? 0.f : m_run;
      float pv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pv[e] = real ? ex2_approx(x[e] - mu) : 0.f;
      l_run += (pv[0] + pv[1]) + (pv[2] + pv[3]);
      const uint32_t pa0 = pack_bf16x2(pv[0], pv[1]);   // P[g][2q, 2q+1]
      const uint32_t pa2 = pack_bf16x2(pv[2], pv[3]);   // P[g][8 + 2q, +1]
      // ---- O (heads x D) += P V, NT n-tiles of 8 columns
#pragma unroll
      for (int j = 0; j < NT / 2; ++j) {
        const int nt = 2 * j + (mi >> 1);          // n-tile of this lane's matrix
        const uint32_t addr = st + kSlab + (nt >> 3) * kBox + v_tok * 128 +
                              (((nt & 7) ^ (v_tok & 7)) << 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(addr, b0, b1, b2, b3);
        mma_bf16(o[2 * j], pa0, 0u, pa2, 0u, b0, b1);
        mma_bf16(o[2 * j + 1], pa0, 0u, pa2, 0u, b2, b3);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));
    }
    gb += nb;
    // The merge below synchronises the 128 compute threads through an mbarrier
    // with bounded waits (never bar.sync): if a warp gave up above, the others
    // give up at their next sync instead of waiting for it forever.
    if (!__all_sync(0xffffffffu, ok)) break;
    // ---- merge the four warps' states (logsumexp rule)
    float lq = l_run;
    lq += __shfl_xor_sync(0xffffffffu, lq, 1);
    lq += __shfl_xor_sync(0xffffffffu, lq, 2);
    if (real && qd == 0) {
      red[warp * kMaxGroup + g] = m_run;
      red[kComputeWarps * kMaxGroup + warp * kMaxGroup + g] = lq;
    }
    if (real) {
#pragma unroll
      for (int n = 0; n < NT; ++n)
        *reinterpret_cast<float2*>(mrg + (warp * kMaxGroup + g) * D + 8 * n + 2 * qd) =
            make_float2(o[n][0], o[n][1]);
    }
    if (!sync128()) break;
    // thread t merges column t % D of heads t / D, t / D + 128 / D, ...
    for (int cell = tid; cell < G * D; cell += kComputeThreads) {
      const int hh = cell / D, dcol = cell % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) M = fmaxf(M, red[w * kMaxGroup + hh]);
      float lt = 0.f, sum = 0.f;
#pragma unroll
      for (int w = 0; w < kComputeWarps; ++w) {
        const float mw = red[w * kMaxGroup + hh];
        const float wgt = (mw == -INFINITY) ? 0.f : ex2_approx(mw - M);
        lt += red[kComputeWarps * kMaxGroup + w * kMaxGroup + hh] * wgt;
        sum += mrg[(w * kMaxGroup + hh) * D + dcol] * wgt;
      }
      const size_t row = (static_cast<size_t>(seq) * a.Hq + kvh * G + hh) * a.max_splits + split;
      a.part_o[row * D + dcol] = sum / lt;
      if (dcol == 0) a.part_l[row] = (M + log2f(lt)) * 0.6931471805599453f;
    }
    if (!sync128()) break;             // red / merge buffer are reused by the next item
  }
}

// One CTA per (query head, sequence), thread = head-dim column.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeArgs a) {
  const int h = blockIdx.x;
  const int seq = blockIdx.y;
  const int dcol = threadIdx.x;
  const int ctx_in = a.context_lens[seq];
  if (ctx_in < 1 || ctx_in > a.max_ctx) {   // outside the documented range: report
    if (h == 0 && dcol == 0) atomicCAS(a.err, 0u, kErrBadIndex + 3);
  }
  const int ctx = max(1, min(ctx_in, a.max_ctx));
  const int nblk = (ctx + kBlk - 1) / kBlk;
  const int ns = (nblk + a.split_blocks - 1) / a.split_blocks;
  const size_t row0 = (static_cast<size_t>(seq) * a.Hq + h) * a.max_splits;
  float mx = -INFINITY;
  for (int s = 0; s < ns; ++s) mx = fmaxf(mx, a.part_l[row0 + s]);
  float wsum = 0.f, acc = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = expf(a.part_l[row0 + s] - mx);
    wsum += w;
    acc = fmaf(w, a.part_o[(row0 + s) * D + dcol], acc);
  }
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);
  o[(static_cast<size_t>(seq) * a.Hq + h) * D + dcol] = __float2bfloat16_rn(acc / wsum);
  if (a.lse != nullptr && dcol == 0)
    a.lse[static_cast<size_t>(seq) * a.Hq + h] = mx + logf(wsum);
}

template <int D>
cudaError_t launch_decode_d(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a,
                            cudaStream_t stream, int dev, int sms) {
  static std::atomic<bool> attr_set[64];   // per device; racing first calls both set it
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DecCfg<D>::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const long long total = static_cast<long long>(a.max_splits) * a.Hkv * a.num_seqs;
  const long long want = 2ll * sms;        // two resident CTAs per SM
  const int g1 = static_cast<int>(total < want ? total : want);
  cudaError_t ez = cudaMemsetAsync(a.counter, 0, sizeof(unsigned int), stream);
  if (ez != cudaSuccess) return ez;
  decode_split_kernel<D><<<g1, kThreads, DecCfg<D>::kSmemBytes, stream>>>(tk, tv, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(a.Hq, a.num_seqs);
  decode_combine_kernel<D><<<g2, D, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

int decode_split_blocks() { return 64; }
int decode_max_group() { return kMaxGroup; }

cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a,
                          cudaStream_t stream) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (a.split_blocks > kMaxSplitBlocks || a.group < 1 || a.group > kMaxGroup)
    return cudaErrorInvalidValue;
  static std::atomic<int> sms[64];
  int n_sm = dev < 64 ? sms[dev].load() : 0;
  if (n_sm == 0) {
    cudaError_t e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    if (dev < 64) sms[dev] = n_sm;
  }
  return a.d == 128 ? launch_decode_d<128>(tk, tv, a, stream, dev, n_sm)
                    : launch_decode_d<64>(tk, tv, a, stream, dev, n_sm);
}

// --------------------------------------------------- allocation-free variant
// Scratch for paged_attn_decode_noalloc: the split partials live in this
// file-scope device array instead of a caller-provided workspace, for callers
// that must not allocate device memory. Every GPU that loads the library holds
// it (kDecodeScratchBytes) until the process exits. All calls share it: calls
// that overlap on the GPU race on it. The launcher clears the work counter
// (the only part that must start at zero) on every call, and the combine
// kernel only reads partials the split kernel of the same call has written.
constexpr size_t kDecodeScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) uint8_t g_decode_scratch[kDecodeScratchBytes];

size_t decode_scratch_bytes() { return kDecodeScratchBytes; }

// Device address of the scratch array on the current device. In host code the
// array's name is only a stand-in, so the address is looked up once per device
// (with that device current) and cached.
cudaError_t decode_scratch_ptr(void** out) {
  static std::atomic<void*> ptrs[64];   // host threads racing on a first call store the same value
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  void* p = ptrs[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    ptrs[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace fa
