// quantize.cu -- per-tensor FP8 e4m3 quantiser with an optional fused
// 128-point Walsh-Hadamard rotation.
//
// [P2] "Zyphra rilascia ZYFA, kernel di attenzione FP8 ottimizzati per le GPU
// AMD" (aicronaca.it), section "Perche l'FP8 non basta da solo": a Hadamard
// rotation of Q and K roughly halves the input quantisation error at ~0.1% of
// the attention time.
//
// Two HBM-bound passes (a per-tensor scale needs the global max first):
//   pass 1  rotate (optional) and reduce max|x| -> workspace (atomicMax on the
//           fp32 bit pattern, order independent, hence deterministic)
//   pass 2  rotate again, scale by fl32(448/amax), round to e4m3 with
//           satfinite, write bytes; one thread writes the descale.
// Layout: each warp owns one 128-channel slice at a time, lane l holding
// channels 4l..4l+3; butterflies at strides 1 and 2 run inside a thread,
// strides 4..64 pair lanes l and l^(stride/4) through shuffles.  Every
// butterfly is the fp32 pair (a+b, a-b) with a the lower channel, so the
// rotation is bit-reproducible.
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "zq_internal.h"

namespace zq {

template <bool BF16IN>
__device__ __forceinline__ void load4(const void* x, int64_t i, float (&v)[4]) {
  if constexpr (BF16IN) {
    uint2 u = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(x) + i);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xFFFF0000u);
  } else {
    float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(x) + i));
    v[0] = f.x;
    v[1] = f.y;
    v[2] = f.z;
    v[3] = f.w;
  }
}

__device__ __forceinline__ void fwht128_warp(float (&v)[4], int lane) {
  float a, b;
  a = v[0]; b = v[1]; v[0] = a + b; v[1] = a - b;  // stride 1
  a = v[2]; b = v[3]; v[2] = a + b; v[3] = a - b;
  a = v[0]; b = v[2]; v[0] = a + b; v[2] = a - b;  // stride 2
  a = v[1]; b = v[3]; v[1] = a + b; v[3] = a - b;
#pragma unroll
  for (int m = 1; m <= 16; m <<= 1) {  // strides 4, 8, 16, 32, 64
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (o - v[i]) : (v[i] + o);
    }
  }
}

template <bool BF16IN, bool HAD>
__global__ void __launch_bounds__(256) quant_amax_kernel(const void* __restrict__ x, int64_t n,
                                                         unsigned* __restrict__ amax_bits) {
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * 4;
  float m = 0.0f;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n; i += stride) {
    float v[4];
    load4<BF16IN>(x, i, v);
    if constexpr (HAD) fwht128_warp(v, lane);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[8];
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
    atomicMax(amax_bits, __float_as_uint(r));
  }
}

template <bool BF16IN, bool HAD>
__global__ void __launch_bounds__(256) quant_write_kernel(const void* __restrict__ x, int64_t n,
                                                          const unsigned* __restrict__ amax_bits,
                                                          uint8_t* __restrict__ out,
                                                          float* __restrict__ descale) {
  const int lane = threadIdx.x & 31;
  const float amax = __uint_as_float(*amax_bits);
  const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    float ds = __fdiv_rn(amax, 448.0f);
    if (HAD) ds = __fmul_rn(ds, 0.08838834764831845f);  // fl32(2^-3.5)
    *descale = ds;
  }
  const int64_t stride = (int64_t)gridDim.x * blockDim.x * 4;
  for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; i < n; i += stride) {
    float v[4];
    load4<BF16IN>(x, i, v);
    if constexpr (HAD) fwht128_warp(v, lane);
    __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)), __NV_SATFINITE, __NV_E4M3);
    __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint32_t*>(out + i) = (uint32_t)lo | ((uint32_t)hi << 16);
  }
}

// ---------------------------------------------------------------------------
// d = 192 with rotation (MLA queries and keys): one warp per 192-channel
// vector.  Lane l holds channels 4l..4l+3 of the 128-slice (rotated by
// fwht128_warp) and channels 128+2l, 128+2l+1 of the 64-slice, rotated by
// H64 (stride 1 inside the thread, strides 2..32 through shuffles) and then
// multiplied by fl32(sqrt 2), so that both slices scale scores by 128.
template <bool BF16IN>
__device__ __forceinline__ void load2(const void* x, int64_t i, float (&v)[2]) {
  if constexpr (BF16IN) {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(static_cast<const uint16_t*>(x) + i);
    v[0] = __uint_as_float(u << 16);
    v[1] = __uint_as_float(u & 0xFFFF0000u);
  } else {
    const float2 f = __ldg(reinterpret_cast<const float2*>(static_cast<const float*>(x) + i));
    v[0] = f.x;
    v[1] = f.y;
  }
}

__device__ __forceinline__ void fwht64x2_warp_scaled(float (&v)[2], int lane) {
  float a = v[0], b = v[1];
  v[0] = a + b;  // stride 1
  v[1] = a - b;
#pragma unroll
  for (int m = 1; m <= 16; m <<= 1) {  // strides 2, 4, 8, 16, 32
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? (o - v[i]) : (v[i] + o);
    }
  }
  v[0] = __fmul_rn(v[0], 1.41421356237309504880f);  // fl32(sqrt 2)
  v[1] = __fmul_rn(v[1], 1.41421356237309504880f);
}

template <bool BF16IN>
__global__ void __launch_bounds__(256) quant192_amax_kernel(const void* __restrict__ x, int64_t n_vec,
                                                            unsigned* __restrict__ amax_bits) {
  const int lane = threadIdx.x & 31;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  float m = 0.0f;
  for (int64_t vec = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); vec < n_vec;
       vec += wstride) {
    float a[4], c[2];
    load4<BF16IN>(x, vec * 192 + 4 * lane, a);
    load2<BF16IN>(x, vec * 192 + 128 + 2 * lane, c);
    fwht128_warp(a, lane);
    fwht64x2_warp_scaled(c, lane);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(a[0]), fabsf(a[1])), fmaxf(fabsf(a[2]), fabsf(a[3]))));
    m = fmaxf(m, fmaxf(fabsf(c[0]), fabsf(c[1])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[8];
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float r = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
    atomicMax(amax_bits, __float_as_uint(r));
  }
}

template <bool BF16IN>
__global__ void __launch_bounds__(256) quant192_write_kernel(const void* __restrict__ x, int64_t n_vec,
                                                             const unsigned* __restrict__ amax_bits,
                                                             uint8_t* __restrict__ out,
                                                             float* __restrict__ descale) {
  const int lane = threadIdx.x & 31;
  const float amax = __uint_as_float(*amax_bits);
  const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0)
    *descale = __fmul_rn(__fdiv_rn(amax, 448.0f), 0.08838834764831845f);  // x fl32(2^-3.5)
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t vec = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); vec < n_vec;
       vec += wstride) {
    float a[4], c[2];
    load4<BF16IN>(x, vec * 192 + 4 * lane, a);
    load2<BF16IN>(x, vec * 192 + 128 + 2 * lane, c);
    fwht128_warp(a, lane);
    fwht64x2_warp_scaled(c, lane);
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(a[0], inv), __fmul_rn(a[1], inv)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(a[2], inv), __fmul_rn(a[3], inv)), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint32_t*>(out + vec * 192 + 4 * lane) = (uint32_t)lo | ((uint32_t)hi << 16);
    const __nv_fp8x2_storage_t t = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(c[0], inv), __fmul_rn(c[1], inv)), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint16_t*>(out + vec * 192 + 128 + 2 * lane) = (uint16_t)t;
  }
}

// ---------------------------------------------------------------------------
// One scale per (batch, group of heads): x is (B, S, H, d) and the heads
// [gi*g, gi*g + g) of batch b share slot b*(H/g) + gi, i.e. the per-(batch,
// kv head) descales of flash_attn_func's FP8 interface.  The grid is
// (chunks, slots): a CTA works inside one slot, so its maximum goes out in
// a single atomicMax on the slot's word.  Each of a slot's S rows holds g*d
// contiguous elements at ((b*S + s)*H + gi*g)*d.
//   HM 0/1  items of 4 elements per thread (row length g*d, a multiple of
//           8).  With the rotation (HM 1, d % 128 == 0) a row is a whole
//           number of 128-slices and a warp's 32 consecutive items are one
//           aligned slice, so fwht128_warp applies unchanged.
//   HM 2    d = 192 with the rotation: one warp per 192-vector (g per row).
// Items are visited by a grid-stride walk within the slot; the (row, item
// in row) position advances by a fixed step without a division per item.
struct ItemWalk {
  int64_t row;
  int col;
  int64_t drow;
  int dcol, ipr;
  __device__ ItemWalk(int64_t k0, int64_t step, int ipr_) : ipr(ipr_) {
    row = k0 / ipr_;
    col = (int)(k0 % ipr_);
    drow = step / ipr_;
    dcol = (int)(step % ipr_);
  }
  __device__ __forceinline__ void next() {
    row += drow;
    col += dcol;
    if (col >= ipr) {
      col -= ipr;
      ++row;
    }
  }
};

struct GroupGeo {
  int64_t S;  // rows per slot
  int H, d, g, gpb;  // heads, channels, heads per slot, slots per batch
};

__device__ __forceinline__ int64_t slot_base(const GroupGeo& G, int slot) {
  const int b = slot / G.gpb, gi = slot % G.gpb;
  return ((int64_t)b * G.S * G.H + (int64_t)gi * G.g) * G.d;
}

__device__ __forceinline__ float block_max_256(float m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
  return r;
}

template <bool BF16IN, int HM>
__global__ void __launch_bounds__(256) quantg_amax_kernel(const void* __restrict__ x, GroupGeo G,
                                                          unsigned* __restrict__ amax_bits) {
  const int lane = threadIdx.x & 31;
  const int slot = blockIdx.y;
  const int64_t base = slot_base(G, slot);
  const int64_t rstride = (int64_t)G.H * G.d;
  float m = 0.0f;
  if constexpr (HM == 2) {
    const int nw = blockDim.x >> 5;
    ItemWalk w((int64_t)blockIdx.x * nw + (threadIdx.x >> 5), (int64_t)gridDim.x * nw, G.g);
    for (; w.row < G.S; w.next()) {
      const int64_t v0 = base + w.row * rstride + (int64_t)w.col * 192;
      float a[4], c[2];
      load4<BF16IN>(x, v0 + 4 * lane, a);
      load2<BF16IN>(x, v0 + 128 + 2 * lane, c);
      fwht128_warp(a, lane);
      fwht64x2_warp_scaled(c, lane);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(a[0]), fabsf(a[1])), fmaxf(fabsf(a[2]), fabsf(a[3]))));
      m = fmaxf(m, fmaxf(fabsf(c[0]), fabsf(c[1])));
    }
  } else {
    ItemWalk w((int64_t)blockIdx.x * blockDim.x + threadIdx.x, (int64_t)gridDim.x * blockDim.x,
               G.g * G.d / 4);
    for (; w.row < G.S; w.next()) {
      float v[4];
      load4<BF16IN>(x, base + w.row * rstride + 4 * (int64_t)w.col, v);
      if constexpr (HM == 1) fwht128_warp(v, lane);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
    }
  }
  const float r = block_max_256(m);
  if (threadIdx.x == 0) atomicMax(amax_bits + slot, __float_as_uint(r));
}

__device__ __forceinline__ uint32_t e4m3x4(const float (&v)[4], float inv) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
      make_float2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv)), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
      make_float2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv)), __NV_SATFINITE, __NV_E4M3);
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

template <bool BF16IN, int HM>
__global__ void __launch_bounds__(256) quantg_write_kernel(const void* __restrict__ x, GroupGeo G,
                                                           const unsigned* __restrict__ amax_bits,
                                                           uint8_t* __restrict__ out,
                                                           float* __restrict__ descale) {
  const int lane = threadIdx.x & 31;
  const int slot = blockIdx.y;
  const float amax = __uint_as_float(amax_bits[slot]);
  const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    float ds = __fdiv_rn(amax, 448.0f);
    if (HM != 0) ds = __fmul_rn(ds, 0.08838834764831845f);  // fl32(2^-3.5)
    descale[slot] = ds;
  }
  const int64_t base = slot_base(G, slot);
  const int64_t rstride = (int64_t)G.H * G.d;
  if constexpr (HM == 2) {
    const int nw = blockDim.x >> 5;
    ItemWalk w((int64_t)blockIdx.x * nw + (threadIdx.x >> 5), (int64_t)gridDim.x * nw, G.g);
    for (; w.row < G.S; w.next()) {
      const int64_t v0 = base + w.row * rstride + (int64_t)w.col * 192;
      float a[4], c[2];
      load4<BF16IN>(x, v0 + 4 * lane, a);
      load2<BF16IN>(x, v0 + 128 + 2 * lane, c);
      fwht128_warp(a, lane);
      fwht64x2_warp_scaled(c, lane);
      *reinterpret_cast<uint32_t*>(out + v0 + 4 * lane) = e4m3x4(a, inv);
      const __nv_fp8x2_storage_t t = __nv_cvt_float2_to_fp8x2(
          make_float2(__fmul_rn(c[0], inv), __fmul_rn(c[1], inv)), __NV_SATFINITE, __NV_E4M3);
      *reinterpret_cast<uint16_t*>(out + v0 + 128 + 2 * lane) = (uint16_t)t;
    }
  } else {
    ItemWalk w((int64_t)blockIdx.x * blockDim.x + threadIdx.x, (int64_t)gridDim.x * blockDim.x,
               G.g * G.d / 4);
    for (; w.row < G.S; w.next()) {
      const int64_t i = base + w.row * rstride + 4 * (int64_t)w.col;
      float v[4];
      load4<BF16IN>(x, i, v);
      if constexpr (HM == 1) fwht128_warp(v, lane);
      *reinterpret_cast<uint32_t*>(out + i) = e4m3x4(v, inv);
    }
  }
}

// Host-side launcher of the grouped quantiser; arguments were validated by
// the caller (B, H >= 1, S >= 0, H % g == 0, B*H/g <= 65535).
cudaError_t launch_quantize_grouped(const void* x, int x_bf16, int B, int64_t S, int H, int d, int g,
                                    int hadamard, void* out, float* descale, void* workspace,
                                    cudaStream_t st, int num_sms) {
  unsigned* amax = static_cast<unsigned*>(workspace);
  GroupGeo G;
  G.S = S;
  G.H = H;
  G.d = d;
  G.g = g;
  G.gpb = H / g;
  const int n_slots = B * G.gpb;
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned) * (size_t)n_slots, st);
  if (e != cudaSuccess) return e;
  const int threads = 256;
  // items per slot, in the unit one thread (HM 0/1) or one warp (HM 2) takes
  const int64_t items = hadamard == 2 ? S * g : S * (int64_t)(g * d / 4);
  const int64_t per_cta = hadamard == 2 ? threads / 32 : threads;
  const int64_t useful = (items + per_cta - 1) / per_cta;
  const int64_t want = ((int64_t)num_sms * 8 + n_slots - 1) / n_slots;
  int cps = (int)(want < useful ? want : useful);
  if (cps < 1) cps = 1;
  const dim3 grid(cps, n_slots);
#define ZQ_QUANTG_LAUNCH(BF, HM_)                                                                 \
  do {                                                                                            \
    quantg_amax_kernel<BF, HM_><<<grid, threads, 0, st>>>(x, G, amax);                            \
    quantg_write_kernel<BF, HM_><<<grid, threads, 0, st>>>(x, G, amax, (uint8_t*)out, descale);   \
  } while (0)
  if (x_bf16) {
    if (hadamard == 2) ZQ_QUANTG_LAUNCH(true, 2);
    else if (hadamard) ZQ_QUANTG_LAUNCH(true, 1);
    else ZQ_QUANTG_LAUNCH(true, 0);
  } else {
    if (hadamard == 2) ZQ_QUANTG_LAUNCH(false, 2);
    else if (hadamard) ZQ_QUANTG_LAUNCH(false, 1);
    else ZQ_QUANTG_LAUNCH(false, 0);
  }
#undef ZQ_QUANTG_LAUNCH
  return cudaGetLastError();
}

// Host-side launcher; arguments were validated by the caller.
cudaError_t launch_quantize(const void* x, int x_bf16, int64_t n, int hadamard, void* out,
                            float* descale, void* workspace, cudaStream_t st, int num_sms) {
  unsigned* amax = static_cast<unsigned*>(workspace);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned), st);
  if (e != cudaSuccess) return e;
  const int threads = 256;
  int64_t cap = (int64_t)num_sms * 8;
  if (hadamard == 2) {  // d = 192: one warp per vector
    const int64_t n_vec = n / 192;
    int64_t want = (n_vec + (threads / 32) - 1) / (threads / 32);
    int blocks = (int)(want < cap ? (want > 0 ? want : 1) : cap);
    if (x_bf16) {
      quant192_amax_kernel<true><<<blocks, threads, 0, st>>>(x, n_vec, amax);
      quant192_write_kernel<true><<<blocks, threads, 0, st>>>(x, n_vec, amax, (uint8_t*)out, descale);
    } else {
      quant192_amax_kernel<false><<<blocks, threads, 0, st>>>(x, n_vec, amax);
      quant192_write_kernel<false><<<blocks, threads, 0, st>>>(x, n_vec, amax, (uint8_t*)out, descale);
    }
    return cudaGetLastError();
  }
  int64_t want = (n / 4 + threads - 1) / threads;
  int blocks = (int)(want < cap ? (want > 0 ? want : 1) : cap);
#define ZQ_QUANT_LAUNCH(BF, HD)                                                               \
  do {                                                                                        \
    quant_amax_kernel<BF, HD><<<blocks, threads, 0, st>>>(x, n, amax);                        \
    quant_write_kernel<BF, HD><<<blocks, threads, 0, st>>>(x, n, amax, (uint8_t*)out, descale); \
  } while (0)
  if (x_bf16) {
    if (hadamard) ZQ_QUANT_LAUNCH(true, true);
    else ZQ_QUANT_LAUNCH(true, false);
  } else {
    if (hadamard) ZQ_QUANT_LAUNCH(false, true);
    else ZQ_QUANT_LAUNCH(false, false);
  }
#undef ZQ_QUANT_LAUNCH
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Several tensors in one pass pair (Q, K and V of an attention call): one
// clear of the amax words, one amax launch and one write launch whose grid
// row blockIdx.y is the tensor.  Each tensor is quantised exactly as by the
// per-tensor kernels above (same per-thread element walk relative to its own
// grid, same fp32 operations), so the bytes and descales are identical.
template <bool BF16IN, bool HAD>
__device__ __forceinline__ float amax_part(const void* x, int64_t n, int64_t t0, int64_t nthreads, int lane) {
  float m = 0.0f;
  for (int64_t i = t0 * 4; i < n; i += nthreads * 4) {
    float v[4];
    load4<BF16IN>(x, i, v);
    if constexpr (HAD) fwht128_warp(v, lane);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
  }
  return m;
}

template <bool BF16IN>
__device__ __forceinline__ float amax192_part(const void* x, int64_t n_vec, int64_t w0, int64_t nwarps, int lane) {
  float m = 0.0f;
  for (int64_t vec = w0; vec < n_vec; vec += nwarps) {
    float a[4], c[2];
    load4<BF16IN>(x, vec * 192 + 4 * lane, a);
    load2<BF16IN>(x, vec * 192 + 128 + 2 * lane, c);
    fwht128_warp(a, lane);
    fwht64x2_warp_scaled(c, lane);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(a[0]), fabsf(a[1])), fmaxf(fabsf(a[2]), fabsf(a[3]))));
    m = fmaxf(m, fmaxf(fabsf(c[0]), fabsf(c[1])));
  }
  return m;
}

// The write pass walks each thread's elements in the reverse order of the
// amax pass: the grid covers the tensor in rounds of nthreads * 4 elements,
// and the rounds the amax pass read last are the likeliest to still sit in
// L2 (the three tensors of a 4K call fit in it).
template <bool BF16IN, bool HAD>
__device__ __forceinline__ void write_part(const void* x, int64_t n, float inv, uint8_t* out, int64_t t0,
                                           int64_t nthreads, int lane) {
  const int64_t step = nthreads * 4;
  if (t0 * 4 >= n) return;
  for (int64_t r = (n - t0 * 4 + step - 1) / step - 1; r >= 0; --r) {
    const int64_t i = t0 * 4 + r * step;
    float v[4];
    load4<BF16IN>(x, i, v);
    if constexpr (HAD) fwht128_warp(v, lane);
    *reinterpret_cast<uint32_t*>(out + i) = e4m3x4(v, inv);
  }
}

template <bool BF16IN>
__device__ __forceinline__ void write192_part(const void* x, int64_t n_vec, float inv, uint8_t* out, int64_t w0,
                                              int64_t nwarps, int lane) {
  if (w0 >= n_vec) return;
  for (int64_t r = (n_vec - w0 + nwarps - 1) / nwarps - 1; r >= 0; --r) {  // reverse rounds, as write_part
    const int64_t vec = w0 + r * nwarps;
    float a[4], c[2];
    load4<BF16IN>(x, vec * 192 + 4 * lane, a);
    load2<BF16IN>(x, vec * 192 + 128 + 2 * lane, c);
    fwht128_warp(a, lane);
    fwht64x2_warp_scaled(c, lane);
    *reinterpret_cast<uint32_t*>(out + vec * 192 + 4 * lane) = e4m3x4(a, inv);
    const __nv_fp8x2_storage_t t = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(c[0], inv), __fmul_rn(c[1], inv)), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint16_t*>(out + vec * 192 + 128 + 2 * lane) = (uint16_t)t;
  }
}

__global__ void __launch_bounds__(256) quant_multi_amax_kernel(QuantItems Q, unsigned* __restrict__ amax_bits) {
  const QuantItem I = Q.it[blockIdx.y];
  const int lane = threadIdx.x & 31;
  // this tensor's own grid: its first `blocks` CTAs of the row
  const int64_t nb = I.blocks;
  float m = 0.0f;
  if ((int64_t)blockIdx.x < nb) {
    if (I.had == 2) {
      const int64_t w0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
      const int64_t nw = nb * (blockDim.x >> 5);
      m = I.bf16 ? amax192_part<true>(I.x, I.n / 192, w0, nw, lane) : amax192_part<false>(I.x, I.n / 192, w0, nw, lane);
    } else {
      const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
      const int64_t nt = nb * blockDim.x;
      if (I.bf16)
        m = I.had ? amax_part<true, true>(I.x, I.n, t0, nt, lane) : amax_part<true, false>(I.x, I.n, t0, nt, lane);
      else
        m = I.had ? amax_part<false, true>(I.x, I.n, t0, nt, lane) : amax_part<false, false>(I.x, I.n, t0, nt, lane);
    }
  }
  const float r = block_max_256(m);
  if (threadIdx.x == 0 && (int64_t)blockIdx.x < nb) atomicMax(amax_bits + blockIdx.y, __float_as_uint(r));
}

__global__ void __launch_bounds__(256) quant_multi_write_kernel(QuantItems Q, const unsigned* __restrict__ amax_bits) {
  const QuantItem I = Q.it[blockIdx.y];
  const int64_t nb = I.blocks;
  if ((int64_t)blockIdx.x >= nb) return;
  const int lane = threadIdx.x & 31;
  const float amax = __uint_as_float(amax_bits[blockIdx.y]);
  const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    float ds = __fdiv_rn(amax, 448.0f);
    if (I.had) ds = __fmul_rn(ds, 0.08838834764831845f);  // fl32(2^-3.5)
    *I.descale = ds;
  }
  if (I.had == 2) {
    const int64_t w0 = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t nw = nb * (blockDim.x >> 5);
    if (I.bf16) write192_part<true>(I.x, I.n / 192, inv, I.out, w0, nw, lane);
    else write192_part<false>(I.x, I.n / 192, inv, I.out, w0, nw, lane);
  } else {
    const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nt = nb * blockDim.x;
    if (I.bf16) {
      if (I.had) write_part<true, true>(I.x, I.n, inv, I.out, t0, nt, lane);
      else write_part<true, false>(I.x, I.n, inv, I.out, t0, nt, lane);
    } else {
      if (I.had) write_part<false, true>(I.x, I.n, inv, I.out, t0, nt, lane);
      else write_part<false, false>(I.x, I.n, inv, I.out, t0, nt, lane);
    }
  }
}

// Blocks of one tensor in the per-tensor launcher below (the same count,
// so that the element walk of every thread is the same).
static int quant_blocks(int64_t n, int hadamard, int num_sms) {
  const int threads = 256;
  const int64_t cap = (int64_t)num_sms * 8;
  const int64_t want = hadamard == 2 ? (n / 192 + (threads / 32) - 1) / (threads / 32) : (n / 4 + threads - 1) / threads;
  return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

cudaError_t launch_quantize_multi(QuantItems Q, int count, void* workspace, cudaStream_t st, int num_sms) {
  unsigned* amax = static_cast<unsigned*>(workspace);
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(unsigned) * (size_t)count, st);
  if (e != cudaSuccess) return e;
  int gx = 1;
  for (int t = 0; t < count; ++t) {
    Q.it[t].blocks = quant_blocks(Q.it[t].n, Q.it[t].had, num_sms);
    if (Q.it[t].blocks > gx) gx = Q.it[t].blocks;
  }
  const dim3 grid(gx, count);
  quant_multi_amax_kernel<<<grid, 256, 0, st>>>(Q, amax);
  quant_multi_write_kernel<<<grid, 256, 0, st>>>(Q, amax);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant.  Some callers cannot hand the library a device
// workspace: hosts whose device memory is owned by another allocator that
// offers no scratch API, and latency-critical serving loops that forbid
// cudaMalloc because it can synchronise the whole device.  For them the
// quantiser's scratch (the amax word) lives in a fixed file-scope device
// array instead.  Every GPU that loads this library keeps the array until
// the process exits.
constexpr size_t kNoAllocScratchBytes = 256;
static __device__ __align__(256) unsigned g_quant_scratch[kNoAllocScratchBytes / sizeof(unsigned)];

// Device address of g_quant_scratch on `dev`, looked up once per device
// (with that device current) and cached.  nullptr on failure.
void* noalloc_scratch_for_device(int dev) {
  constexpr int kMaxDevices = 64;
  static void* cache[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  void* p = __atomic_load_n(&cache[dev], __ATOMIC_ACQUIRE);
  if (p) return p;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_quant_scratch) != cudaSuccess || !ptr) return nullptr;
  __atomic_store_n(&cache[dev], ptr, __ATOMIC_RELEASE);
  return ptr;
}

size_t noalloc_scratch_capacity() { return kNoAllocScratchBytes; }

}  // namespace zq
