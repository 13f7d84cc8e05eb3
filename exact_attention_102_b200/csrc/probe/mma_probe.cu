// mma_probe.cu — a measurement tool, never linked into libfa.so: SM cycles
// per tcgen05.mma (kind::f16, M = 128, K = 16, bf16 operands, fp32
// accumulate) for one N and one operand form, issued back to back by one
// thread of each CTA (one CTA per SM), so that the time per MMA is the
// tensor core's time on that shape. The operands are zeros: only the shape
// and where the operands live matter for the time.
//   form 0 (SS): A and B in shared memory, K-major, 128-byte swizzle
//   form 1 (TS): A in TMEM (two bf16 per column), B in shared memory
// Built and run by exact_attention_102_b200.probe_mma.
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "prim.cuh"

namespace {
constexpr int kThreads = 128;
constexpr int kABytes = 128 * 128;         // A: 128 rows x 64 bf16 (one 128 B chunk per row)
constexpr int kBBytes = 256 * 128;         // B: up to 256 rows x 64 bf16
// the request (not the use) is 200 KB, so that one CTA holds an SM and its TMEM
constexpr int kSmem = 200 * 1024;
static_assert(kABytes + kBBytes + 1024 + 64 <= kSmem, "probe shared memory");
constexpr uint32_t kCols = 512;            // D [0, 256), A (form 1) [256, 288)

// Templated on the form and N, and issued in unrolled groups of 8 from fixed
// descriptors, like the kernels' own product groups: a runtime branch or
// descriptor arithmetic between two MMAs of one issuing thread costs more
// than the MMA itself.
template <int TS, int N>
__global__ void __launch_bounds__(kThreads, 1)
probe_kernel(int iters, unsigned long long* cycles, uint32_t* err) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t a_addr = fa::smem_u32(sm), b_addr = a_addr + kABytes;
  const uint32_t bar = b_addr + kBBytes;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kABytes + kBBytes + 8);
  for (int i = threadIdx.x; i < (kABytes + kBBytes) / 16; i += kThreads)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    fa::mbar_init(bar, 1);
    fa::fence_mbar_init();
  }
  if (threadIdx.x < 32) {
    fa::tmem_alloc(fa::smem_u32(tmem_slot), kCols);
    fa::tmem_relinquish();
  }
  fa::fence_async_smem();
  fa::tc_fence_before();
  __syncthreads();
  fa::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    constexpr uint32_t id = fa::idesc_f16(128, N, 1, 0, 0);
    const uint64_t da = fa::smem_desc_sw128(a_addr, 16, 1024);
    const uint64_t db = fa::smem_desc_sw128(b_addr, 16, 1024);
    uint32_t phase = 0;
    bool ok = true;
    // one round to warm up, one timed
    for (int round = 0; round < 2 && ok; ++round) {
      const unsigned long long t0 = clock64();
      for (int i = 0; i < iters; i += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int kk = u & 3;              // K = 16 steps inside the 128 B chunk
          if constexpr (TS)
            fa::umma_f16_ts(tmem, tmem + 256 + kk * 8, db + kk * 2, id, 1u);
          else
            fa::umma_f16_ss(tmem, da + kk * 2, db + kk * 2, id, 1u);
        }
      }
      fa::umma_commit(bar);
      ok = fa::mbar_wait(bar, phase, err, 1, nullptr);
      const unsigned long long t1 = clock64();
      if (ok) {
        phase ^= 1;
        if (round == 1) cycles[blockIdx.x] = t1 - t0;
      }
    }
    // a wait that gave up: let the products in flight finish (bounded) before
    // the columns are freed
    if (!ok) fa::mbar_wait(bar, phase, nullptr, 1, nullptr, 100000000ull);
  }
  fa::tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    fa::tc_fence_after();
    fa::tmem_dealloc(tmem, kCols);
  }
}
}  // namespace

// Runs the probe on `ctas` CTAs of the current device and copies each CTA's
// cycle count for `iters` MMAs into host_cycles[ctas]. Returns 0, or 1 for
// bad arguments, 2 for a CUDA error, 3 when a wait gave up.
extern "C" __attribute__((visibility("default"))) int mma_probe(int ts, int n, int iters, int ctas,
                                                               unsigned long long* host_cycles) {
  if ((n != 64 && n != 128 && n != 256) || iters < 8 || iters > (1 << 16) || iters % 8 != 0 ||
      ctas < 1 || ctas > 1024 || host_cycles == nullptr || (ts != 0 && ts != 1))
    return 1;
  void (*kern)(int, unsigned long long*, uint32_t*) =
      ts ? (n == 64 ? probe_kernel<1, 64> : n == 128 ? probe_kernel<1, 128> : probe_kernel<1, 256>)
         : (n == 64 ? probe_kernel<0, 64> : n == 128 ? probe_kernel<0, 128> : probe_kernel<0, 256>);
  unsigned long long* d_cycles = nullptr;
  uint32_t* d_err = nullptr;
  if (cudaMalloc(&d_cycles, sizeof(unsigned long long) * ctas) != cudaSuccess) return 2;
  if (cudaMalloc(&d_err, sizeof(uint32_t)) != cudaSuccess) {
    cudaFree(d_cycles);
    return 2;
  }
  int rc = 0;
  uint32_t h_err = 0;
  if (cudaMemset(d_err, 0, sizeof(uint32_t)) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess) {
    rc = 2;
  } else {
    kern<<<ctas, kThreads, kSmem>>>(iters, d_cycles, d_err);
    if (cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(host_cycles, d_cycles, sizeof(unsigned long long) * ctas,
                   cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(&h_err, d_err, sizeof(uint32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
      rc = 2;
    else if (h_err != 0)
      rc = 3;
  }
  cudaFree(d_cycles);
  cudaFree(d_err);
  return rc;
}
