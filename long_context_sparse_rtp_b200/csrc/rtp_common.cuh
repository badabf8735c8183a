// rtp_common.cuh -- device helpers shared by the RTPurbo kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rtp.h"

namespace rtp {

constexpr int kD = 128;          // head dimension d_h
constexpr int kR = 16;           // indexer dimension r
constexpr int kMaxHeads = 256;   // query heads per layer supported
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Workspace status block (first 256 bytes of every workspace).
struct DevStatus {
  int32_t code;    // 0 = ok, RTP_ERR_DEVICE_TIMEOUT when a bounded wait gave up
  int32_t where;   // kernel id that set it
  int32_t pad[62];
};
constexpr size_t kStatusBytes = 256;

// Head roles, passed by value to kernels.
struct HeadMap {
  int32_t H, Hkv, G;
  int32_t n_ret;                 // retrieval query heads (slots hr)
  int32_t n_rkv;                 // retrieval kv heads
  int32_t n_loc;                 // local query heads
  int32_t n_lkv;                 // local kv heads
  int32_t H_k16;                 // k16 head slots
  int16_t ret_q[kMaxHeads];      // hr -> query head
  int16_t ret_k16[kMaxHeads];    // hr -> k16 slot
  int16_t rkv[kMaxHeads];        // retrieval kv rank -> kv head
  int16_t lkv[kMaxHeads];        // local kv rank -> kv head
};

// ------------------------------------------------------------------ bf16
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ------------------------------------------------------------------ mma.sync
// D = A(16x16 bf16, row) * B(16x8 bf16, col) + C (fp32).
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4],
                                         uint32_t b0, uint32_t b1, const float (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%11,%12,%13};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]),
        "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// ------------------------------------------------------------------ cp.async
__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gmem, bool pred) {
  const int sz = pred ? 16 : 0;  // 0 -> zero-fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr),
               "l"(gmem), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// ------------------------------------------------------------------ misc
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float quad_max(float v) {
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
  v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
  return v;
}
__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

// Softmax mass w in [0, 1] as unsigned fixed point with 40 fractional bits,
// truncating.  Integer sums of these are exact and order-independent, which
// keeps every top-p decision deterministic.
__device__ __forceinline__ unsigned long long mass_fixed40(float w) {
  const uint32_t b = __float_as_uint(w);
  if (b >= 0x3F800000u) return 1ull << 40;  // w >= 1 (or inf / nan): saturate at 1
  const int e = int(b >> 23) & 0xFF;
  if (e == 0) return 0ull;  // zero / subnormal: below 2^-126
  const unsigned long long m = (b & 0x7FFFFFu) | 0x800000u;
  const int sh = e - 110;   // w = m * 2^(e-150); fixed = m * 2^(e-110)
  if (sh >= 0) return m << sh;
  if (sh > -24) return m >> (-sh);
  return 0ull;
}
constexpr double kFixedOne = 1099511627776.0;  // 2^40

// max(a, b, c) in one instruction (exact, like two fmaxf).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// Two fp32 lanes in one 64-bit register: packed arithmetic, one instruction for
// both lanes, each lane rounded as the scalar operation with the same rounding
// mode would round it.
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};\n" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;\n" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;\n" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2_add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2_sub(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2_add_rm(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rm.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2_add_rz(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rz.f32x2 %0, %1, %2;\n" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Order-preserving map of an fp32 score to uint32 (larger score -> larger key).
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// A kernel launched with launch_dependent: wait until the previous kernel on the
// stream has completed and its writes are visible (no-op for a plain launch).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

__device__ __forceinline__ void set_status(DevStatus* st, int code, int where) {
  if (st != nullptr) {
    atomicCAS(&st->code, 0, code);
    st->where = where;
  }
}

}  // namespace rtp
