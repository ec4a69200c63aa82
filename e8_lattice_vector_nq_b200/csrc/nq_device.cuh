// nq_device.cuh -- device-side helpers shared by the libnq kernels (sm_100a):
// cp.async, bulk and TMA tensor copies in inline PTX, bf16 unpacking, packed
// fp32x2 arithmetic and the device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nq {

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kRowPad = 272;  // smem bytes per staged 128 x bf16 row (256 + 16: conflict-free)
constexpr int kTileSlots = 32;

// fp32 constants of the scale rule: C = 1/sqrt(128), G_b = 1/(A_b sqrt(128))
// with A_3 = 3.5, A_2 = 1.5, each the fp32 nearest to the real number.
constexpr uint32_t kCBits = 0x3DB504F3u;
constexpr uint32_t kG3Bits = 0x3CCEE116u;
constexpr uint32_t kG2Bits = 0x3D715BEFu;
constexpr float kMagicRound = 12582912.0f;  // 1.5 * 2^23: x + M - M = rint(x) for |x| < 2^22
constexpr float kTwo23 = 8388608.0f;        // 2^23: bits(2^23 + j) = 0x4B000000 | j

// Device error word of this translation unit, reserved for in-kernel
// failure reports; read and cleared through the ABI (nq_device_error).
static __device__ unsigned int g_nq_error;

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------- bulk async copies
// shared -> global, tracked by this thread's bulk groups.
__device__ __forceinline__ void bulk_s2g(void* gmem_dst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gmem_dst),
               "r"(smem_u32(smem_src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until this thread's committed bulk stores have finished READING smem.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until this thread's committed bulk stores are complete (globally visible).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Per-thread 16-byte async copy global -> shared (LDGSTS), grouped by
// commit/wait; each thread waits only for its own groups.
__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// TMA tensor store of a 4-D box from shared memory, tracked by bulk groups.
__device__ __forceinline__ void tma_store_4d(const void* tmap, uint32_t smem_src, int x, int y,
                                             int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          tmap),
      "r"(smem_src), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// Make this thread's generic-proxy smem writes visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------- conversions
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ float4 lds128f(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// a * b + c (low 32 bits) in one instruction; packing a code at a bit offset
// k is mad_u32(code, 1 << k, word) (a shift-and-add for a power-of-two b).
__device__ __forceinline__ uint32_t mad_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// ----------------------------------------------------- packed fp32 pairs
// IEEE round-to-nearest per lane (sm_100 f32x2 instructions).
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  // a - b == fma(b, -1, a): one rounding of the exact difference.
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

}  // namespace nq
