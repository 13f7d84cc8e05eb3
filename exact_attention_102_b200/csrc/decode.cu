// decode.cu — single-token attention over a paged KV cache (memory bound).
//
// "FlashAttention系列优化" (johneyzheng.top), section PagedAttention: the KV
// cache of a sequence lives in fixed-size physical blocks reached through a
// per-sequence block table; several sequences (parallel sampling) may point
// at the same physical block. The kernel only follows the table.
//
// Work split: one CTA per (sequence, KV head, split of `split_blocks`
// 16-token blocks). A CTA serves the 4 query heads that share its KV head, so
// every K/V byte is read from HBM once per query group. Each split produces a
// partial (O_s normalised over its own keys, L_s = its logsumexp); the
// combine kernel merges the splits with L = log sum_s exp(L_s),
// O = sum_s exp(L_s - L) O_s, which follows from the definition of the
// logsumexp statistic (91haoming.cn repost, "前向傳播改進").
//
// Inside a split CTA:
//   warp 4 (producer)  loads the split's slice of the block table, then copies
//                      each (block, KV head) K and V slab (16 x 128 bf16 =
//                      4 KB each, contiguous) into an 8-stage shared-memory
//                      ring with untiled bulk copies (no multicast), one full /
//                      empty mbarrier pair per stage.
//   warps 0..3         thread (t, c) = (tid / 8, tid % 8) owns token slot t of
//                      every block and head-dim elements [8c, 8c+8) and
//                      [64+8c, 64+8c+8): 16-byte shared loads, 64 FMAs for the
//                      4 heads' scores, a 3-step shuffle reduction over the 8
//                      threads of the slot, an online-softmax update per slot
//                      (running max with rescale skipping, running sum), then
//                      64 FMAs into the slot's unnormalised output. At the end
//                      the 16 slot states are merged through shared memory
//                      with the same logsumexp rule.
#include "prim.cuh"
#include "kernels.h"

namespace fa {

namespace {

constexpr int kD = 128;
constexpr int kBlk = 16;          // tokens per physical block
constexpr int kGroup = 4;         // query heads per KV head
constexpr int kStages = 8;
constexpr int kSlab = kBlk * kD * 2;           // bytes of one (block, kv head) K or V slab
constexpr int kStageBytes = 2 * kSlab;         // K + V
constexpr int kMaxSplitBlocks = 128;
constexpr int kComputeThreads = 128;
constexpr int kThreads = kComputeThreads + 32;
constexpr float kRescaleThreshold = 8.0f;

// shared memory layout (bytes)
constexpr int kRingOff = 0;
constexpr int kTableOff = kRingOff + kStages * kStageBytes;
constexpr int kBarOff = kTableOff + kMaxSplitBlocks * 4;
constexpr int kMiscOff = kBarOff + 2 * kStages * 8;
constexpr int kRedOff = kMiscOff + 16;     // cross-warp reduction scratch: [4 warps][4 heads] x 2
constexpr int kSmemBytes = kRedOff + 2 * 16 * 4 + 128;

enum : uint32_t { kSiteFull = 0x21, kSiteEmpty = 0x22, kSiteDrain = 0x23 };

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16);
  f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16);
  f[7] = __uint_as_float(u.w & 0xffff0000u);
}

__global__ void __launch_bounds__(kThreads, 2) decode_split_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int split = blockIdx.x;
  const int kvh = blockIdx.y;
  const int seq = blockIdx.z;
  int ctx = a.context_lens[seq];
  ctx = max(1, min(ctx, a.max_ctx));
  const int nblk = (ctx + kBlk - 1) / kBlk;
  const int first = split * a.split_blocks;
  if (first >= nblk) return;  // this split is past the sequence's end
  const int nb = min(nblk - first, a.split_blocks);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t sbase = smem_u32(smem);
  int* table = reinterpret_cast<int*>(smem + kTableOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kMiscOff);
  auto full = [&](int s) -> uint32_t { return sbase + kBarOff + 8 * s; };
  auto empty = [&](int s) -> uint32_t { return sbase + kBarOff + 8 * (kStages + s); };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), kComputeThreads / 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    const int* trow = a.block_table + static_cast<size_t>(seq) * a.max_blocks + first;
    for (int i = lane; i < nb; i += 32) {
      int id = trow[i];
      if (id < 0 || id >= a.num_phys) {  // never dereference a bad id
        atomicCAS(a.err, 0u, kErrBadIndex + 1);
        id = 0;
      }
      table[i] = id;
    }
    __syncwarp();
    if (lane == 0) {
      const uint8_t* kc = static_cast<const uint8_t*>(a.k_cache);
      const uint8_t* vc = static_cast<const uint8_t*>(a.v_cache);
      int issued = 0;
      for (int i = 0; i < nb; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(empty(s), ((i / kStages) & 1) ^ 1, a.err, kSiteEmpty, abort_flag)) break;
        const size_t slab = (static_cast<size_t>(table[i]) * a.Hkv + kvh) * kSlab;
        mbar_arrive_expect_tx(full(s), kStageBytes);
        bulk_load(sbase + kRingOff + s * kStageBytes, kc + slab, kSlab, full(s));
        bulk_load(sbase + kRingOff + s * kStageBytes + kSlab, vc + slab, kSlab, full(s));
        ++issued;
      }
      for (int i = max(0, issued - kStages); i < issued; ++i)
        mbar_wait(full(i % kStages), (i / kStages) & 1, a.err, kSiteDrain, nullptr, 200000000ull);
    }
    return;
  }

  // -------------------------------------------------------------- compute
  const int t = tid >> 3;   // token slot 0..15
  const int c = tid & 7;    // element group
  const int h0 = kvh * kGroup;
  float qv[kGroup][16];
  {
    const __nv_bfloat16* qp =
        static_cast<const __nv_bfloat16*>(a.q) + (static_cast<size_t>(seq) * a.Hq + h0) * kD;
#pragma unroll
    for (int hh = 0; hh < kGroup; ++hh) {
      const uint4 u0 = *reinterpret_cast<const uint4*>(qp + hh * kD + 8 * c);
      const uint4 u1 = *reinterpret_cast<const uint4*>(qp + hh * kD + 64 + 8 * c);
      float f0[8], f1[8];
      bf16x8_to_f32(u0, f0);
      bf16x8_to_f32(u1, f1);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        qv[hh][e] = f0[e] * a.scale_log2;  // scores come out in exp2 units
        qv[hh][8 + e] = f1[e] * a.scale_log2;
      }
    }
  }
  float m[kGroup], l[kGroup], acc[kGroup][16];
#pragma unroll
  for (int hh = 0; hh < kGroup; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[hh][e] = 0.f;
  }

  bool ok = true;
  for (int i = 0; i < nb; ++i) {
    const int s = i % kStages;
    ok = __all_sync(0xffffffffu,
                    mbar_wait(full(s), (i / kStages) & 1, a.err, kSiteFull, abort_flag));
    if (!ok) break;
    const uint8_t* kst = smem + kRingOff + s * kStageBytes + t * (kD * 2);
    float kf[16];
    {
      const uint4 u0 = *reinterpret_cast<const uint4*>(kst + 16 * c);
      const uint4 u1 = *reinterpret_cast<const uint4*>(kst + 128 + 16 * c);
      float f0[8], f1[8];
      bf16x8_to_f32(u0, f0);
      bf16x8_to_f32(u1, f1);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        kf[e] = f0[e];
        kf[8 + e] = f1[e];
      }
    }
    float x[kGroup];
#pragma unroll
    for (int hh = 0; hh < kGroup; ++hh) {
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        s0 = fmaf(qv[hh][e], kf[e], s0);
        s1 = fmaf(qv[hh][e + 1], kf[e + 1], s1);
      }
      x[hh] = s0 + s1;
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
#pragma unroll
      for (int hh = 0; hh < kGroup; ++hh) x[hh] += __shfl_xor_sync(0xffffffffu, x[hh], o);
    }
    const bool valid = (first + i) * kBlk + t < ctx;
    float p[kGroup];
#pragma unroll
    for (int hh = 0; hh < kGroup; ++hh) {
      if (valid && x[hh] > m[hh] + kRescaleThreshold) {
        const float alpha = ex2_approx(m[hh] - x[hh]);  // 0 while m = -inf
        m[hh] = x[hh];
        l[hh] *= alpha;
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[hh][e] *= alpha;
      }
      p[hh] = valid ? ex2_approx(x[hh] - m[hh]) : 0.f;
      l[hh] += p[hh];
    }
    const uint8_t* vst = kst + kSlab;
    {
      const uint4 u0 = *reinterpret_cast<const uint4*>(vst + 16 * c);
      const uint4 u1 = *reinterpret_cast<const uint4*>(vst + 128 + 16 * c);
      float f0[8], f1[8];
      bf16x8_to_f32(u0, f0);
      bf16x8_to_f32(u1, f1);
#pragma unroll
      for (int hh = 0; hh < kGroup; ++hh) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc[hh][e] = fmaf(p[hh], f0[e], acc[hh][e]);
          acc[hh][8 + e] = fmaf(p[hh], f1[e], acc[hh][8 + e]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));
  }

  // ---- merge the 16 token-slot states (same logsumexp rule as the combine)
  float* red = reinterpret_cast<float*>(smem + kRedOff);   // [2][4 warps][4 heads]
  float mw[kGroup];
#pragma unroll
  for (int hh = 0; hh < kGroup; ++hh) {
    float v = m[hh];
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
    mw[hh] = v;
  }
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < kGroup; ++hh) red[warp * 4 + hh] = mw[hh];
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  float M[kGroup], w[kGroup];
#pragma unroll
  for (int hh = 0; hh < kGroup; ++hh) {
    M[hh] = fmaxf(fmaxf(red[hh], red[4 + hh]), fmaxf(red[8 + hh], red[12 + hh]));
    w[hh] = (m[hh] == -INFINITY) ? 0.f : ex2_approx(m[hh] - M[hh]);
    float lv = l[hh] * w[hh];
    lv += __shfl_xor_sync(0xffffffffu, lv, 8);
    lv += __shfl_xor_sync(0xffffffffu, lv, 16);
    mw[hh] = lv;
  }
  if (lane == 0) {
#pragma unroll
    for (int hh = 0; hh < kGroup; ++hh) red[16 + warp * 4 + hh] = mw[hh];
  }
  // every stage has been consumed: the ring can hold the [16 slots][4][128] sums
  float* slot = reinterpret_cast<float*>(smem + kRingOff);
#pragma unroll
  for (int hh = 0; hh < kGroup; ++hh) {
    float4* dst0 = reinterpret_cast<float4*>(slot + (t * kGroup + hh) * kD + 8 * c);
    float4* dst1 = reinterpret_cast<float4*>(slot + (t * kGroup + hh) * kD + 64 + 8 * c);
    const float ww = w[hh];
    dst0[0] = make_float4(acc[hh][0] * ww, acc[hh][1] * ww, acc[hh][2] * ww, acc[hh][3] * ww);
    dst0[1] = make_float4(acc[hh][4] * ww, acc[hh][5] * ww, acc[hh][6] * ww, acc[hh][7] * ww);
    dst1[0] = make_float4(acc[hh][8] * ww, acc[hh][9] * ww, acc[hh][10] * ww, acc[hh][11] * ww);
    dst1[1] = make_float4(acc[hh][12] * ww, acc[hh][13] * ww, acc[hh][14] * ww, acc[hh][15] * ww);
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
  if (!ok) return;
  const int dcol = tid;  // 0..127
#pragma unroll
  for (int hh = 0; hh < kGroup; ++hh) {
    const float lt = red[16 + hh] + red[20 + hh] + red[24 + hh] + red[28 + hh];
    float sum = 0.f;
#pragma unroll
    for (int ts = 0; ts < kBlk; ++ts) sum += slot[(ts * kGroup + hh) * kD + dcol];
    const size_t row = (static_cast<size_t>(seq) * a.Hq + h0 + hh) * a.max_splits + split;
    a.part_o[row * kD + dcol] = sum / lt;
    if (dcol == 0) a.part_l[row] = (M[hh] + log2f(lt)) * 0.6931471805599453f;
  }
}

__global__ void __launch_bounds__(128) decode_combine_kernel(DecodeArgs a) {
  const int h = blockIdx.x;
  const int seq = blockIdx.y;
  const int dcol = threadIdx.x;
  int ctx = a.context_lens[seq];
  ctx = max(1, min(ctx, a.max_ctx));
  const int nblk = (ctx + kBlk - 1) / kBlk;
  const int ns = (nblk + a.split_blocks - 1) / a.split_blocks;
  const size_t row0 = (static_cast<size_t>(seq) * a.Hq + h) * a.max_splits;
  float mx = -INFINITY;
  for (int s = 0; s < ns; ++s) mx = fmaxf(mx, a.part_l[row0 + s]);
  float wsum = 0.f, acc = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = expf(a.part_l[row0 + s] - mx);
    wsum += w;
    acc = fmaf(w, a.part_o[(row0 + s) * kD + dcol], acc);
  }
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(a.o);
  o[(static_cast<size_t>(seq) * a.Hq + h) * kD + dcol] = __float2bfloat16_rn(acc / wsum);
  if (a.lse != nullptr && dcol == 0)
    a.lse[static_cast<size_t>(seq) * a.Hq + h] = mx + logf(wsum);
}

}  // namespace

int decode_split_blocks() { return 64; }

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  if (a.split_blocks > kMaxSplitBlocks) return cudaErrorInvalidValue;
  dim3 g1(a.max_splits, a.Hkv, a.num_seqs);
  decode_split_kernel<<<g1, kThreads, kSmemBytes, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(a.Hq, a.num_seqs);
  decode_combine_kernel<<<g2, kD, 0, stream>>>(a);
  return cudaGetLastError();
}

// --------------------------------------------------- allocation-free variant
// Scratch for paged_attn_decode_noalloc: the split partials live in this
// file-scope device array instead of a caller-provided workspace, for callers
// that must not allocate device memory. Every GPU that loads the library holds
// it (kDecodeScratchBytes) until the process exits. All calls share it: calls
// that overlap on the GPU race on it. Nothing needs clearing between calls,
// because the combine kernel only reads partials the split kernel of the same
// call has just written.
constexpr size_t kDecodeScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) uint8_t g_decode_scratch[kDecodeScratchBytes];

size_t decode_scratch_bytes() { return kDecodeScratchBytes; }

// Device address of the scratch array on the current device. In host code the
// array's name is only a stand-in, so the address is looked up once per device
// (with that device current) and cached.
cudaError_t decode_scratch_ptr(void** out) {
  static void* ptrs[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    ptrs[dev] = p;
  }
  *out = ptrs[dev];
  return cudaSuccess;
}

}  // namespace fa
