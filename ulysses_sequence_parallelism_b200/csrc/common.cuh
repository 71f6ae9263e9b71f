// Shared device helpers for the Ulysses B200 kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#define ULY_DEV __device__ __forceinline__

namespace uly {

constexpr int kMaxRanks = 16;

// Per-rank pointer tables, passed by value as kernel parameters.
struct RankPtrs {
  const void* p[kMaxRanks];
};
struct RankPtrsMut {
  void* p[kMaxRanks];
};
struct RankPtrsF {
  float* p[kMaxRanks];
};
struct RankPtrsFC {
  const float* p[kMaxRanks];
};

// Library-wide device error word (bounded waits that gave up, bounds checks).
// Bit layout: [31:24] kernel id, [23:0] site-specific detail. The library is
// one translation unit, so these are defined here.
__device__ uint32_t g_error_word = 0;
// Poll cap for every bounded device-side wait (0 = the kernel's default).
__device__ uint32_t g_wait_limit = 0;

enum ErrKernel : uint32_t { kErrFwd = 1u, kErrBwd = 2u, kErrPermute = 3u };

ULY_DEV void report_error(uint32_t kernel, uint32_t detail) {
  atomicCAS(&g_error_word, 0u, (kernel << 24) | (detail & 0xFFFFFFu));
}

// ----------------------------------------------------------------- small math
ULY_DEV float ex2_approx(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Three-input fp32 max (one instruction on sm_100).
ULY_DEV float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Packed fp32 pair arithmetic (sm_100 f32x2): two lanes of work per instruction.
// (d0, d1) = (a0 * s + c, a1 * s + c)
ULY_DEV void ffma2_sc(float& d0, float& d1, float a0, float a1, float s, float c) {
  asm("{\n\t.reg .b64 a, b, c, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %4};\n\tmov.b64 c, {%5, %5};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(s), "f"(c));
}
// (acc0, acc1) += (a0, a1)
ULY_DEV void fadd2_acc(float& acc0, float& acc1, float a0, float a1) {
  asm("{\n\t.reg .b64 a, b, d;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "add.rn.f32x2 d, a, b;\n\tmov.b64 {%0, %1}, d;\n\t}"
      : "=f"(acc0), "=f"(acc1)
      : "f"(acc0), "f"(acc1), "f"(a0), "f"(a1));
}

ULY_DEV uint32_t pack_bf16x2(float lo, float hi) {
  // cvt.rn.bf16x2.f32 d, a, b puts a in the upper half and b in the lower half.
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// First token of the document containing row i (cu_seqlens may be null).
// Clamped into [0, i] whatever the array holds.
ULY_DEV int doc_start_of(const int32_t* __restrict__ cu, int num_seqs, int i) {
  if (cu == nullptr) return 0;
  int lo = 0, hi = num_seqs;  // find the last m with cu[m] <= i
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= i) lo = mid; else hi = mid - 1;
  }
  int s = __ldg(cu + lo);
  return s < 0 ? 0 : (s > i ? i : s);
}

// One past the last token of the document containing row i, clamped into [i+1, N].
ULY_DEV int doc_end_of(const int32_t* __restrict__ cu, int num_seqs, int i, int N) {
  if (cu == nullptr) return N;
  int lo = 0, hi = num_seqs;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= i) lo = mid; else hi = mid - 1;
  }
  int e = (lo + 1 <= num_seqs) ? __ldg(cu + lo + 1) : N;
  return e <= i ? i + 1 : (e > N ? N : e);
}

// ----------------------------------------------------------------- addresses
ULY_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

}  // namespace uly
