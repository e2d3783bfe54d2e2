// Shared device helpers for the GPT-2 training-step kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

typedef __nv_bfloat16 bf16;

// Device-side error word, read by the host at sync points.  Kernels never trap: a
// failed check records a code here and the kernel skips the offending access.
enum DeviceError : int {
  DEVERR_NONE = 0,
  DEVERR_TOKEN = 1,     // input token id outside [0, vocab_size)
  DEVERR_TARGET = 2,    // target outside [0, vocab_size) and not the ignore index -1
  DEVERR_TIMEOUT = 3,   // a bounded wait on an mbarrier gave up
  DEVERR_INTERNAL = 4,
};

extern __device__ int g_device_error;

__device__ __forceinline__ void raise_device_error(int code) {
  atomicCAS(&g_device_error, 0, code);
}

// ---------------------------------------------------------------- conversions
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<bf16> {
  static __device__ __forceinline__ float to_f(bf16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ bf16 from_f(float x) { return __float2bfloat16_rn(x); }
};

template <typename T> __device__ __forceinline__ float ld_f(const T* p) { return Elem<T>::to_f(*p); }
template <typename T> __device__ __forceinline__ void st_f(T* p, float v) { *p = Elem<T>::from_f(v); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(h);
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Column sums of one warp's 32 rows of 16 values (x[j] = row `lane`, column j): lane l returns
// the sum of column l >> 1 (lanes l and l ^ 1 agree).  Each step halves the values a lane
// keeps, adding its partner's half: 8 + 4 + 2 + 1 shuffles, then one for the last pair.
__device__ __forceinline__ float warp_colsum16(float (&x)[16], int lane) {
#pragma unroll
  for (int s = 16, n = 16; s >= 2; s >>= 1, n >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = upper ? x[j] : x[j + n / 2];
      const float keep = upper ? x[j + n / 2] : x[j];
      x[j] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return x[0] + __shfl_xor_sync(0xffffffffu, x[0], 1);
}

// ---------------------------------------------------------------- GELU (tanh form)
// gelu(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))  -- the approximation GPT-2
// used ("Karpathy's Zero to Hero, Lecture 9" notes, section "1:48:25 – 2:00:19").
// tanhf is CUDA's, called, not re-implemented.
#define GELU_A 0.7978845608028654f
#define GELU_C 0.044715f
__device__ __forceinline__ float gelu_tanh_f(float x) {
  float t = tanhf(GELU_A * (x + GELU_C * x * x * x));
  return 0.5f * x * (1.0f + t);
}
__device__ __forceinline__ float gelu_tanh_grad_f(float x) {
  float t = tanhf(GELU_A * (x + GELU_C * x * x * x));
  return 0.5f * (1.0f + t) + 0.5f * x * (1.0f - t * t) * GELU_A * (1.0f + 3.0f * GELU_C * x * x);
}

// Same formulas with the hardware tanh approximation (tanh.approx.f32, relative error
// about 2^-11), used where the result is rounded to bf16 anyway.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float gelu_tanh_fast(float x) {
  const float t = tanh_approx(GELU_A * (x + GELU_C * x * x * x));
  return 0.5f * x * (1.0f + t);
}
__device__ __forceinline__ float gelu_tanh_grad_fast(float x) {
  const float t = tanh_approx(GELU_A * (x + GELU_C * x * x * x));
  return 0.5f * (1.0f + t) + 0.5f * x * (1.0f - t * t) * GELU_A * (1.0f + 3.0f * GELU_C * x * x);
}

// gelu(x) and gelu'(x) together from one tanh, in fp32 (tanhf) and with the hardware tanh
// approximation (results rounded to bf16).
__device__ __forceinline__ void gelu_tanh_and_grad_f(float x, float& g, float& gp) {
  const float t = tanhf(GELU_A * (x + GELU_C * x * x * x));
  g = 0.5f * x * (1.0f + t);
  gp = 0.5f * (1.0f + t) + 0.5f * x * (1.0f - t * t) * GELU_A * (1.0f + 3.0f * GELU_C * x * x);
}
__device__ __forceinline__ void gelu_tanh_and_grad_fast(float x, float& g, float& gp) {
  const float t = tanh_approx(GELU_A * (x + GELU_C * x * x * x));
  g = 0.5f * x * (1.0f + t);
  gp = 0.5f * (1.0f + t) + 0.5f * x * (1.0f - t * t) * GELU_A * (1.0f + 3.0f * GELU_C * x * x);
}

// ---------------------------------------------------------------- single PTX instructions
// 2^x by the hardware approximation (ex2.approx.ftz; subnormal results flushed to zero),
// the 3-input maximum of sm_100, and paired fp32 arithmetic.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Paired fp32 arithmetic (one instruction for two lanes of data): a*b+c and a+b.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

// gelu(x) and gelu'(x) for two values with paired fp32 arithmetic and the hardware tanh
// (results rounded to bf16).  With p = (1 + t) / 2 and t = tanh(A x (1 + C x^2)):
//   gelu(x) = x p,   gelu'(x) = p + (x / 2) A (1 - t^2)(1 + 3 C x^2) = p (1 + x A (1 - t)(1 + 3 C x^2)),
// using 1 - t^2 = (1 - t)(1 + t): eleven paired operations and two tanh per pair.
__device__ __forceinline__ void gelu2_and_grad_fast(float2 x, float2& g, float2& gp) {
  const float2 one = make_float2(1.0f, 1.0f), half = make_float2(0.5f, 0.5f);
  const float2 x2 = fmul2(x, x);
  const float2 xa = fmul2(x, make_float2(GELU_A, GELU_A));
  const float2 arg = fmul2(xa, ffma2(x2, make_float2(GELU_C, GELU_C), one));
  const float2 t = make_float2(tanh_approx(arg.x), tanh_approx(arg.y));
  const float2 p = ffma2(t, half, half);
  g = fmul2(x, p);
  const float2 omt = ffma2(t, make_float2(-1.0f, -1.0f), one);
  const float2 d = ffma2(x2, make_float2(3.0f * GELU_C, 3.0f * GELU_C), one);
  gp = fmul2(p, ffma2(fmul2(xa, omt), d, one));
}

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ long long cdivll(long long a, long long b) { return (a + b - 1) / b; }
