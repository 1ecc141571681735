// attn_math.cuh -- pieces shared by the attention kernels: the softmax
// arithmetic (exp2 forms, Lean P helpers, e4m3 / bf16 packing, the block
// reference-exponent rule), a cycle counter for the debug trace, and the
// host-side TMA tensor-map encoder for (B, S, H, d) tensors.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace zq {

constexpr int kInvalidExp = -(1 << 20);

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// (a0, a1) * b + c on the paired fp32 FMA path
__device__ __forceinline__ void ffma2(float& r0, float& r1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 x, y, z;\n\t"
      "mov.b64 x, {%2, %3};\n\tmov.b64 y, {%4, %4};\n\tmov.b64 z, {%5, %5};\n\t"
      "fma.rn.f32x2 x, x, y, z;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
// Software 2^z for a pair of values (offloads the MUFU unit).  Cody-Waite
// style reduction z = n + f with n = rne(z) (magic-constant add) and
// f in [-1/2, 1/2], a minimax polynomial p(f) ~ 2^f fitted by the Remez
// exchange (bf16_causal_prefill_02_b200/csrc/exp2_poly_fit.py; max relative
// error 7.5e-5 for degree 3, 2.7e-6 for degree 4), and 2^n applied by adding
// n to the exponent bits.  z is clamped at -126 first (results below 2^-126
// are irrelevant here: they round to 0 in e4m3 and vanish against the row
// sum in bf16).
template <int DEG>
__device__ __forceinline__ void exp2_poly_x2(float& r0, float& r1, float z0, float z1) {
  z0 = fmaxf(z0, -126.0f);
  z1 = fmaxf(z1, -126.0f);
  const float magic = 12582912.0f;  // 1.5 * 2^23
  float t0, t1, f0, f1, p0, p1;
  asm("{\n\t.reg .b64 z, t, n, m;\n\t"
      "mov.b64 z, {%4, %5};\n\tmov.b64 m, {%6, %6};\n\t"
      "add.rn.f32x2 t, z, m;\n\tsub.rn.f32x2 n, t, m;\n\tsub.rn.f32x2 z, z, n;\n\t"
      "mov.b64 {%0, %1}, t;\n\tmov.b64 {%2, %3}, z;\n\t}"
      : "=f"(t0), "=f"(t1), "=f"(f0), "=f"(f1)
      : "f"(z0), "f"(z1), "f"(magic));
  if constexpr (DEG == 3) {
    ffma2(p0, p1, f0, f1, 5.517166853e-02f, 2.426111251e-01f);
    asm("{\n\t.reg .b64 p, f, c;\n\tmov.b64 p, {%0, %1};\n\tmov.b64 f, {%2, %3};\n\t"
        "mov.b64 c, {%4, %4};\n\tfma.rn.f32x2 p, p, f, c;\n\tmov.b64 c, {%5, %5};\n\t"
        "fma.rn.f32x2 p, p, f, c;\n\tmov.b64 {%0, %1}, p;\n\t}"
        : "+f"(p0), "+f"(p1)
        : "f"(f0), "f"(f1), "f"(6.932609677e-01f), "f"(9.999280572e-01f));
  } else {
    ffma2(p0, p1, f0, f1, 9.570102207e-03f, 5.591785908e-02f);
    asm("{\n\t.reg .b64 p, f, c;\n\tmov.b64 p, {%0, %1};\n\tmov.b64 f, {%2, %3};\n\t"
        "mov.b64 c, {%4, %4};\n\tfma.rn.f32x2 p, p, f, c;\n\tmov.b64 c, {%5, %5};\n\t"
        "fma.rn.f32x2 p, p, f, c;\n\tmov.b64 c, {%6, %6};\n\tfma.rn.f32x2 p, p, f, c;\n\t"
        "mov.b64 {%0, %1}, p;\n\t}"
        : "+f"(p0), "+f"(p1)
        : "f"(f0), "f"(f1), "f"(2.402474433e-01f), "f"(6.931217909e-01f), "f"(9.999992847e-01f));
  }
  r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_e4m3x4(float p0, float p1, float p2, float p3) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(p2, p3), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}
__device__ __forceinline__ float pow2i(int e) {  // exact 2^e for -126 <= e <= 127
  return __int_as_float((e + 127) << 23);
}
// Max of 64 floats with four independent 3-input max chains.
// (Lean P and the exact mode take one power-of-2 exponent per 64-key block.)
__device__ __forceinline__ float max64(const float* s) {
  float m0 = fmaxf(s[0], s[1]), m1 = fmaxf(s[2], s[3]);
  float m2 = fmaxf(s[4], s[5]), m3 = fmaxf(s[6], s[7]);
#pragma unroll
  for (int c = 8; c < 64; c += 8) {
    m0 = max3(m0, s[c], s[c + 1]);
    m1 = max3(m1, s[c + 2], s[c + 3]);
    m2 = max3(m2, s[c + 4], s[c + 5]);
    m3 = max3(m3, s[c + 6], s[c + 7]);
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}
// Reference-exponent rule (FP8): the row's exponent E after seeing this
// tile's largest block exponent `emax`; it only moves up, and only when a
// block exceeds it by more than `thr`.
__device__ __forceinline__ int next_ref(int eref_old, int emax, int thr) {
  if (emax <= kInvalidExp) return eref_old;
  if (eref_old <= kInvalidExp) return emax;
  return emax > eref_old + thr ? emax : eref_old;
}

__device__ __forceinline__ uint64_t clk64() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%clock64;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's encoder, looked up once and cached.  Callers on several host
// threads may race to the first lookup: the cache is atomic, and every
// thread stores the same pointer.  A failed lookup is retried on the next
// call.
static inline EncodeTiledFn get_encode_fn() {
  static std::atomic<EncodeTiledFn> cache{nullptr};
  EncodeTiledFn fn = cache.load(std::memory_order_acquire);
  if (fn) return fn;
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  fn = reinterpret_cast<EncodeTiledFn>(ptr);
  cache.store(fn, std::memory_order_release);
  return fn;
}

// Tensor (B, S, H, d) of `es`-byte elements; box = `box_elems` channels x 1
// head x `box_rows` rows x 1 batch.
static inline bool make_map(CUtensorMap* m, const void* base, int es, int B, int S, int H, int d,
                            int box_elems, CUtensorMapSwizzle sw, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * es, (cuuint64_t)H * d * es, (cuuint64_t)S * H * d * es};
  cuuint32_t box[4] = {(cuuint32_t)box_elems, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 4,
                   const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace zq
