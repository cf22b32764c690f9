// kda_common.cuh — shared device helpers of the KDA CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kda.h"

namespace kda {

// ---------------------------------------------------------------------------------------------
// Per-device status word. Kernels OR a kda_status_t bit pattern into it when they detect a fault
// that the host could not see (bad cu_seqlens contents, a bounded wait that gave up); the host
// reads and clears it in kda_last_device_error(). File-scope __device__ storage is instantiated
// once per device context, so there is one word per GPU.
// ---------------------------------------------------------------------------------------------
__device__ unsigned int g_status = 0;  // one definition: the library is a single TU

enum : unsigned int {
  kStatusBadSeqlens = 1u << 0,  // also: a state index beyond the pool
  kStatusTimeout = 1u << 1,
  kStatusBounds = 1u << 2,      // bounds-checked build: an access outside its buffer, skipped
};

__device__ __forceinline__ void raise_status(unsigned int bits) { atomicOr(&g_status, bits); }

// ---------------------------------------------------------------------------------------------
// Bounds-checked build (compiled with KDA_BOUNDS_CHECK, `_build.build(checked=True)`): every entry
// point registers the byte extent of each buffer of its call in a device table (on the call's
// stream, before its launches), and the prefill, decode and recurrent-mode kernels test each
// global access against the extent of the buffer it belongs to. An access outside is skipped — a
// load yields zeros, a bulk copy is left out of its barrier's byte count — and the status word
// gets kStatusBounds, which kda_last_device_error reports as KDA_ERR_INVALID_ARG: a substitute
// for a memory checker that never faults the GPU. The table is one per device, so calls that
// overlap on the GPU would see each other's extents: the checked build runs one call at a time.
// In the normal build the checks compile away.
// ---------------------------------------------------------------------------------------------
enum BufRole : int {
  kBufQ = 0, kBufK, kBufV, kBufLogAlpha, kBufBeta, kBufInitial, kBufFinal, kBufO, kBufWork,
  kBufCuSeqlens, kBufState, kBufIndices, kBufGate, kBufDtBias, kBufALog, kBufNormW,
  // the backward's cotangents in and gradients out
  kBufDO, kBufDFinal, kBufDQ, kBufDK, kBufDV, kBufDLogAlpha, kBufDBeta, kBufDInitial, kBufRoles
};
struct BoundsTable {
  const void* base[kBufRoles];
  unsigned long long bytes[kBufRoles];
};
#ifdef KDA_BOUNDS_CHECK
__device__ BoundsTable g_bounds;
// The table travels as a kernel parameter (captured by value when the call is recorded in a CUDA
// graph, unlike a copy from the caller's stack).
__global__ void set_bounds_kernel(BoundsTable t) { g_bounds = t; }
__device__ __forceinline__ bool in_bounds(int role, const void* p, unsigned long long n) {
  const char* b = static_cast<const char*>(g_bounds.base[role]);
  const char* c = static_cast<const char*>(p);
  if (b != nullptr && c >= b && (unsigned long long)(c - b) + n <= g_bounds.bytes[role])
    return true;
  raise_status(kStatusBounds);
  return false;
}
#define KDA_IN_BOUNDS(role, p, n) (::kda::in_bounds((role), (p), (n)))
// Rows r0 .. r1 - 1 of a row-strided array (row r at p + r * stride elements, D elements each) lie
// in the buffer when its first and its last row do: the rows in between lie between them.
template <typename T>
__device__ __forceinline__ bool rows_in_bounds(int role, const T* p, long long r0, long long r1,
                                               size_t stride, size_t D) {
  return r1 <= r0 || (in_bounds(role, p + (size_t)r0 * stride, D * sizeof(T)) &&
                      in_bounds(role, p + (size_t)(r1 - 1) * stride, D * sizeof(T)));
}
// appends "&& the check" to a condition; nothing at all in the normal build, so that a kernel's
// normal code is exactly what it is without the checks
#define KDA_AND_IN_BOUNDS(role, p, n) && ::kda::in_bounds((role), (p), (n))
constexpr bool kBoundsChecked = true;
#else
#define KDA_IN_BOUNDS(role, p, n) ((void)(p), true)
#define KDA_AND_IN_BOUNDS(role, p, n)
constexpr bool kBoundsChecked = false;
#endif

// ---------------------------------------------------------------------------------------------
// Element access for the two input dtypes.
// ---------------------------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// log(1 + exp(x)) without overflow.
__device__ __forceinline__ float softplus_f(float x) { return x > 20.f ? x : log1pf(expf(x)); }
// 1 / (1 + exp(-x)); exp(-x) = inf for very negative x gives exactly 0.
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + __expf(-x)); }
__host__ __device__ __forceinline__ size_t align_up(size_t x, size_t a) {
  return (x + a - 1) / a * a;
}

// ---------------------------------------------------------------------------------------------
// Sequence / chunk geometry of one prefill call.
//   Without cu_seqlens: sequence n is batch row n, tokens [n*T, (n+1)*T), ceil(T/C) chunks each.
//   With cu_seqlens: chunk_off[n] (device, in the workspace) is the index of the first chunk of
//   sequence n; chunk_off[N] is the number of chunks. A global chunk index is mapped back to its
//   sequence by binary search over chunk_off.
// ---------------------------------------------------------------------------------------------
struct SeqGeometry {
  const int32_t* cu_seqlens;  // device, or nullptr
  const int32_t* chunk_off;   // device [N+1], valid when cu_seqlens != nullptr
  const int32_t* valid;       // device flag written by the chunk-map kernel (varlen only)
  int32_t N;
  int32_t T;  // tokens per sequence when cu_seqlens == nullptr
  int32_t C;
  // device [N], or nullptr: sequence indices by decreasing chunk count (packed varlen batches),
  // so that kernels whose work per sequence is a serial chain start the longest chains first
  const int32_t* order = nullptr;

  __device__ __forceinline__ bool ok() const { return cu_seqlens == nullptr || *valid != 0; }

  __device__ __forceinline__ int num_chunks_total() const {
    return cu_seqlens ? chunk_off[N] : N * ceil_div(T, C);
  }
  __device__ __forceinline__ int seq_begin(int n) const {
    return cu_seqlens ? cu_seqlens[n] : n * T;
  }
  __device__ __forceinline__ int seq_end(int n) const {
    return cu_seqlens ? cu_seqlens[n + 1] : (n + 1) * T;
  }
  __device__ __forceinline__ int first_chunk(int n) const {
    return cu_seqlens ? chunk_off[n] : n * ceil_div(T, C);
  }
  // Sequence at position `i` of the longest-first order (the identity without one).
  __device__ __forceinline__ int seq_at_rank(int i) const { return order ? order[i] : i; }
  // Sequence that owns global chunk `c` (c < num_chunks_total()).
  __device__ __forceinline__ int seq_of_chunk(int c) const {
    if (!cu_seqlens) return c / ceil_div(T, C);
    int lo = 0, hi = N - 1;  // largest n with chunk_off[n] <= c (skips empty sequences)
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (chunk_off[mid] <= c)
        lo = mid;
      else
        hi = mid - 1;
    }
    return lo;
  }
};

// ---------------------------------------------------------------------------------------------
// Asynchronous 16-byte global -> shared copies (cp.async, L2 only) in commit groups: a thread
// waits for its own groups; a barrier after the wait makes every thread's copies visible.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void cp_async_16B(void* dst_smem, const void* src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst_smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// waits until at most `pending` of this thread's most recent groups are still in flight
template <int pending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(pending) : "memory");
}

// ---------------------------------------------------------------------------------------------
// 16-byte vectors of the input dtype into fp32 shared memory (4 floats, or 8 from bf16).
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void store_vec(float* p, uint4 u, float) {
  *reinterpret_cast<float4*>(p) = make_float4(__uint_as_float(u.x), __uint_as_float(u.y),
                                              __uint_as_float(u.z), __uint_as_float(u.w));
}
__device__ __forceinline__ void store_vec(float* p, uint4 u, __nv_bfloat16) {
  *reinterpret_cast<float4*>(p) =
      make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                  __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
  *reinterpret_cast<float4*>(p + 4) =
      make_float4(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xffff0000u),
                  __uint_as_float(u.w << 16), __uint_as_float(u.w & 0xffff0000u));
}

// Rows of Tin (row r at src + r * stride; D a multiple of 16 / sizeof(Tin); 16-byte aligned
// rows) into fp32 shared-memory rows of pitch ld (a multiple of 4), rows >= L as zeros: each
// thread keeps four 16-byte loads in flight before converting them.
template <typename Tin>
__device__ __forceinline__ void stage_rows_f32(float* dst, int ld, const Tin* src, size_t stride,
                                               int rows, int L, int D, int tid, int nt) {
  constexpr int kPer = 16 / sizeof(Tin);
  const int vpr = D / kPer, total = rows * vpr;
  for (int base = 0; base < total; base += 4 * nt) {
    uint4 x[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int idx = base + m * nt + tid, r = idx / vpr, c = idx - r * vpr;
      x[m] = (idx < total && r < L)
                 ? __ldg(reinterpret_cast<const uint4*>(src + r * stride + c * kPer))
                 : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int idx = base + m * nt + tid, r = idx / vpr, c = idx - r * vpr;
      if (idx < total) store_vec(dst + r * ld + c * kPer, x[m], Tin());
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Packed fp32 pairs (mov/fma/mul .f32x2, sm_100a): one issued instruction works on two values,
// each rounded exactly as the scalar operation would round it.
// ---------------------------------------------------------------------------------------------
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 f2_pack(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(f32x2 v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// acc[0..3] += s * b on two packed pairs (each element rounded as fmaf rounds it)
__device__ __forceinline__ void fma_s4(float s, float4 b, float (&acc)[4]) {
  const f32x2 ss = f2_pack(s, s);
  const float2 lo = f2_unpack(f2_fma(ss, f2_pack(b.x, b.y), f2_pack(acc[0], acc[1])));
  const float2 hi = f2_unpack(f2_fma(ss, f2_pack(b.z, b.w), f2_pack(acc[2], acc[3])));
  acc[0] = lo.x;
  acc[1] = lo.y;
  acc[2] = hi.x;
  acc[3] = hi.y;
}

}  // namespace kda
