// Shared device helpers for the JSSA decode-step kernels (sm_100a).
//
// Inline-PTX wrappers for the data-movement and matrix instructions the kernels use:
// 1-D bulk async copies (TMA engine) completing on mbarriers, cp.async 16-byte
// copies, ldmatrix / movmatrix, and the warp-level bf16 MMA.  Every wait on an
// mbarrier is bounded in time and reports a timeout through the device status word.
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

namespace jssa {

// Bits of the device status word (kept in the caller's workspace).
enum : int {
  DEVFLAG_BAD_SEQ_LEN = 1,   // seq_lens[b] outside [0, T_cap] (clamped)
  DEVFLAG_BAD_INDEX = 2,     // an index outside the candidate range (skipped)
  DEVFLAG_BAD_NSEL = 4,      // n_sel outside [0, k] (clamped)
  DEVFLAG_TIMEOUT = 8,       // a bounded wait gave up
};

__device__ __forceinline__ void flag_error(int* status, int bit) {
  if (status) atomicOr(status, bit);
}

// Default limit of a bounded wait, and the one-shot test of the bounded waits that
// jssa_test_withhold_copy() arms in the words after the status word: word 1 = 1 asks the
// first CTA of row 0 of the next selection launch to withhold one bulk copy, word 2 is that
// CTA's wait limit in microseconds.  The CTA disarms word 1 once it has read it.
constexpr uint64_t kWaitLimitNs = 1000000000ull;
struct WaitTest {
  bool withhold;
  uint64_t limit_ns;
};
__device__ __forceinline__ WaitTest wait_test_read(const int* status, bool first_cta) {
  WaitTest t{false, kWaitLimitNs};
  if (status && first_cta) {
    const volatile int* w = status;
    if (w[1] == 1) {
      t.withhold = true;
      const int us = w[2];
      t.limit_ns = static_cast<uint64_t>(us > 0 ? us : 1) * 1000ull;
    }
  }
  return t;
}
__device__ __forceinline__ void wait_test_disarm(int* status) {
  if (status) *reinterpret_cast<volatile int*>(status + 1) = 0;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for the phase with the given parity to complete, for at most `limit_ns`.
// Returns false (and raises DEVFLAG_TIMEOUT) when the limit is reached.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* status,
                                                  uint64_t limit_ns = 1000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      flag_error(status, DEVFLAG_TIMEOUT);
      return false;
    }
  }
}

// 1-D bulk copy global -> shared through the TMA engine; completion is signalled on
// `bar` as transaction bytes.  dst, src and bytes must be multiples of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ------------------------------------------------------------------ cp.async (16 B)
// src_bytes = 0 fills the 16 destination bytes with zeros without reading memory.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ warp matrix ops
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// Round a double to bf16, nearest with ties to even, in a single rounding step.
// Written from the IEEE binary-format definition: bf16 keeps the fp32 exponent
// range and 7 stored fraction bits; below 2^-126 its spacing is 2^-133.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  const uint16_t sign = static_cast<uint16_t>((u >> 48) & 0x8000u);
  const unsigned long long a = u & 0x7FFFFFFFFFFFFFFFull;
  if (a >= 0x7FF0000000000000ull) return (a > 0x7FF0000000000000ull) ? uint16_t(0x7FC0) : uint16_t(sign | 0x7F80);
  const int e = static_cast<int>(a >> 52) - 1023;
  if (e >= -126) {
    unsigned long long keep = a >> 45;  // exponent and the top 7 fraction bits
    const unsigned long long rem = a & ((1ull << 45) - 1);
    const unsigned long long half = 1ull << 44;
    if (rem > half || (rem == half && (keep & 1ull))) keep += 1;
    const double r = __longlong_as_double(static_cast<long long>(keep << 45));
    if (r >= 0x1p128) return uint16_t(sign | 0x7F80);
    return uint16_t(sign | (__float_as_uint(static_cast<float>(r)) >> 16));
  }
  const double q = rint(__longlong_as_double(static_cast<long long>(a)) * 0x1p133);  // whole quanta of 2^-133
  return uint16_t(sign | static_cast<uint16_t>(q));
}

// fp64 -> FP8 E4M3 (the OCP format: bias 7, 3 fraction bits, subnormals in steps of
// 2^-9, largest finite 448 = 0x7E, 0x7F NaN), nearest with ties to even, saturated to
// +-448 (infinities too).  Worked on the bits of the double: a result of 2^-6 or more keeps
// the exponent and the top 3 fraction bits and rounds on the 49 bits below (a carry out of
// the fraction steps the exponent, which is the right code); a smaller one counts whole
// 2^-9 quanta (a count of 8 is the code of 2^-6).
__device__ __forceinline__ uint8_t f64_to_e4m3_rne_sat(double x) {
  const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  const uint8_t sign = static_cast<uint8_t>((u >> 56) & 0x80u);
  const unsigned long long a = u & 0x7FFFFFFFFFFFFFFFull;
  if (a > 0x7FF0000000000000ull) return static_cast<uint8_t>(sign | 0x7Fu);   // NaN
  if (a >= 0x407C000000000000ull) return static_cast<uint8_t>(sign | 0x7Eu);  // |x| >= 448
  const int e = static_cast<int>(a >> 52) - 1023;
  const unsigned long long m = (a & ((1ull << 52) - 1)) | (1ull << 52);
  if (e >= -6) {
    const unsigned long long rem = m & ((1ull << 49) - 1), half = 1ull << 48;
    const uint32_t f = static_cast<uint32_t>(m >> 49) & 7u;
    uint32_t code = (static_cast<uint32_t>(e + 7) << 3) | f;
    if (rem > half || (rem == half && (f & 1u))) code += 1;
    return static_cast<uint8_t>(sign | code);
  }
  const int sh = 43 - e;  // |x| / 2^-9 = m * 2^-sh
  if (sh >= 54) return sign;  // |x| <= 2^-10: rounds to zero (2^-10 itself is a tie to 0)
  uint32_t q = static_cast<uint32_t>(m >> sh);
  const unsigned long long rem = m & ((1ull << sh) - 1), half = 1ull << (sh - 1);
  if (rem > half || (rem == half && (q & 1u))) q += 1;
  return static_cast<uint8_t>(sign | q);
}

// Rotation of a scan thread's 16-byte Kp vectors: VPT vectors per thread, read in the order
// (j + rot) % VPT, so that each 8-thread phase of a 16-byte shared-memory load covers 8
// different 16-byte bank groups for every row size the scans use (rows of 1, 2, 4 or 8
// vectors with one or two threads per token).
template <int VPT>
__device__ __forceinline__ int kp_vector_rotation(int tid) {
  if constexpr (VPT == 1) return 0;
  else if constexpr (VPT == 2) return (tid >> 2) & 1;
  else return (tid >> 1) & 3;
}

// Sum of a thread's per-vector partial dot products, read in the rotated order above
// (a[j] belongs to vector (j + rot) % VPT).  The pairing (a0 + a2) + (a1 + a3) is the same
// fp32 value for every rotation, because each of its additions is commutative; so two
// tokens with identical projected rows get bit-identical scores whichever threads score
// them, and an exact tie stays exact (the lower position then wins the selection).
template <int VPT>
__device__ __forceinline__ float kp_rotated_sum(const float (&a)[VPT]) {
  static_assert(VPT == 1 || VPT == 2 || VPT == 4, "1, 2 or 4 vectors per thread");
  if constexpr (VPT == 1) return a[0];
  else if constexpr (VPT == 2) return a[0] + a[1];
  else return (a[0] + a[2]) + (a[1] + a[3]);
}

// Dot product of one 16-byte vector of a projected-key row with the matching slice of the
// projected query (fp32), the products added in element order.  bf16: 8 elements, widened by
// a shift.  E4M3: 16 elements (element 0 in the lowest byte), each pair widened exactly to
// f16x2 by the hardware conversion and then to fp32.
template <bool F8>
__device__ __forceinline__ float kp_vector_dot(const float* q, uint4 raw) {
  if constexpr (!F8) {
    float x = q[0] * __uint_as_float(raw.x << 16);
    x = fmaf(q[1], __uint_as_float(raw.x & 0xFFFF0000u), x);
    x = fmaf(q[2], __uint_as_float(raw.y << 16), x);
    x = fmaf(q[3], __uint_as_float(raw.y & 0xFFFF0000u), x);
    x = fmaf(q[4], __uint_as_float(raw.z << 16), x);
    x = fmaf(q[5], __uint_as_float(raw.z & 0xFFFF0000u), x);
    x = fmaf(q[6], __uint_as_float(raw.w << 16), x);
    x = fmaf(q[7], __uint_as_float(raw.w & 0xFFFF0000u), x);
    return x;
  } else {
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    float x = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu), __NV_E4M3);
      const float2 f = __half22float2(__half2(hr));
      x = (i == 0) ? q[0] * f.x : fmaf(q[2 * i], f.x, x);
      x = fmaf(q[2 * i + 1], f.y, x);
    }
    return x;
  }
}

// Order-preserving map of an fp32 value to uint32 (larger value -> larger key);
// -0.0 and +0.0 map to the same key.
__device__ __forceinline__ uint32_t float_to_ordered(float f) {
  uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// Launch with an optional 1-D thread-block cluster (cluster_x > 0).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  int n = 0;
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Raise a kernel's dynamic shared memory limit once per device (host side).  `done` is a
// per-kernel table owned by the caller (a function-local static).
template <typename Kernel>
inline cudaError_t set_smem_limit_once(Kernel kernel, size_t bytes, int (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (done[dev] >= static_cast<int>(bytes)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
  if (e == cudaSuccess) done[dev] = static_cast<int>(bytes);
  return e;
}

}  // namespace jssa
