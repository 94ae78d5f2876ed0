// Activation quantisation (per-token FP8, MXFP8, NVFP4) and exact decode of
// quantised activations to bf16.
//
// The pages name the activation formats ("Announcing Humming", sections
// "W8A8 / W4A8 / W4A4" and the MoE activation override in its usage section:
// tokenwise FP8, MXFP8, NVFP4) without a recipe; the recipes here are the
// OCP MX v1.0 shared-exponent rule for MXFP8, amax/448 for per-token FP8 and
// NVIDIA's two-level NVFP4 scheme, with every fp32 step an IEEE operation
// (explicit _rn intrinsics) and every narrowing conversion a hardware
// round-to-nearest-even saturating cvt.
#include <cuda_bf16.h>

#include "hq_internal.cuh"

namespace hq {

// ---- conversions -----------------------------------------------------------

// Two fp32 -> packed E4M3x2 (lo in bits 0..7, hi in bits 8..15), RNE, satfinite.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two fp32 -> packed E2M1x2 (lo in bits 0..3, hi in bits 4..7), RNE, satfinite.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tmov.b32 %0, {t, t, t, t};\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r & 0xFFu;
}

// E4M3 code -> fp32 (exact).  Exponent/mantissa bits are moved into the fp32
// fields and rescaled by 2^120 (the bias difference 127 - 7), which also maps
// E4M3 subnormals onto fp32 subnormals exactly.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const float mag = __uint_as_float((c & 0x7Fu) << 20) * 1.329227995784916e36f;  // 2^120
  return (c & 0x80u) ? -mag : mag;
}

// E2M1 code -> fp32 (exact): 2^(e-1) (1 + m/2), subnormal 0.5 m.
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
  const float mag = __uint_as_float((c & 0x7u) << 22) * 8.507059173023462e37f;  // 2^126
  return (c & 0x8u) ? -mag : mag;
}

// 2^e as fp32 for e in [-127, 127] (2^-127 is a subnormal).
__device__ __forceinline__ float exp2i(int e) {
  return (e >= -126) ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(1u << 22);
}

// floor(log2(a)) for finite a > 0, exact for normal and subnormal fp32.
__device__ __forceinline__ int floor_log2(float a) {
  const uint32_t b = __float_as_uint(a);
  const int ex = (int)((b >> 23) & 0xFF);
  if (ex != 0) return ex - 127;
  return -149 + (31 - __clz((int)(b & 0x7FFFFF)));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---- per-token FP8 ---------------------------------------------------------
// One CTA per row.
__global__ void quant_fp8_token_kernel(int M, int K, const uint16_t *__restrict__ x, uint8_t *__restrict__ q,
                                       float *__restrict__ scales) {
  const int m = blockIdx.x;
  const uint4 *row = reinterpret_cast<const uint4 *>(x + (size_t)m * K);
  const int nv = K / 8;
  float amax = 0.f;
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const uint4 v = row[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
  }
  __shared__ float red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x < 32) {
    float a = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (threadIdx.x == 0) red[0] = a;
  }
  __syncthreads();
  amax = red[0];
  const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f);
  if (threadIdx.x == 0) scales[m] = s;
  uint2 *out = reinterpret_cast<uint2 *>(q + (size_t)m * K);
  for (int i = threadIdx.x; i < nv; i += blockDim.x) {
    const uint4 v = row[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t a = f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(w[2 * j]), s), __fdiv_rn(bf16_hi(w[2 * j]), s));
      const uint32_t b =
          f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(w[2 * j + 1]), s), __fdiv_rn(bf16_hi(w[2 * j + 1]), s));
      o[j] = a | (b << 16);
    }
    out[i] = make_uint2(o[0], o[1]);
  }
}

// ---- FP8 per token and 128 k ------------------------------------------------
// One warp per (row, 128-k group), 4 values per lane: s = amax / 448 (1 for
// an all-zero group), q = e4m3(x / s), as the per-token recipe on each group.
__global__ void quant_fp8_group_kernel(size_t ngroups, const uint16_t *__restrict__ x, uint8_t *__restrict__ q,
                                       float *__restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const size_t warps = (size_t)gridDim.x * (blockDim.x >> 5);
  for (size_t g = blockIdx.x * (size_t)(blockDim.x >> 5) + (threadIdx.x >> 5); g < ngroups; g += warps) {
    const uint2 v = reinterpret_cast<const uint2 *>(x + g * 128)[lane];
    const float f[4] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y)};
    float amax = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f);
    const uint32_t a = f32x2_to_e4m3x2(__fdiv_rn(f[0], s), __fdiv_rn(f[1], s));
    const uint32_t b = f32x2_to_e4m3x2(__fdiv_rn(f[2], s), __fdiv_rn(f[3], s));
    reinterpret_cast<uint32_t *>(q + g * 128)[lane] = a | (b << 16);
    if (lane == 0) scales[g] = s;
  }
}

// ---- MXFP8 -----------------------------------------------------------------
// One thread per 32-element block.
__global__ void quant_mxfp8_kernel(size_t nblocks, const uint16_t *__restrict__ x, uint8_t *__restrict__ q,
                                   uint8_t *__restrict__ scales) {
  for (size_t b = blockIdx.x * (size_t)blockDim.x + threadIdx.x; b < nblocks; b += (size_t)gridDim.x * blockDim.x) {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + b * 32);
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 v = src[i];
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
    int e = 0;
    if (amax > 0.f) {
      e = floor_log2(amax) - 8;
      e = max(-127, min(127, e));
    }
    scales[b] = (uint8_t)(e + 127);
    const float mul = exp2i(-e);
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t a = f32x2_to_e4m3x2(__fmul_rn(bf16_lo(w[2 * i]), mul), __fmul_rn(bf16_hi(w[2 * i]), mul));
      const uint32_t c =
          f32x2_to_e4m3x2(__fmul_rn(bf16_lo(w[2 * i + 1]), mul), __fmul_rn(bf16_hi(w[2 * i + 1]), mul));
      o[i] = a | (c << 16);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(q + b * 32);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// ---- NVFP4 -----------------------------------------------------------------
// Pass 1: tensor amax as the maximum fp32 bit pattern of |x| (non-negative
// floats order like their bit patterns).
__global__ void amax_kernel(size_t n8, const uint16_t *__restrict__ x, unsigned int *__restrict__ amax_bits) {
  float a = 0.f;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4 *>(x)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) a = fmaxf(a, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0 && a > 0.f) atomicMax(amax_bits, __float_as_uint(a));
}

// Pass 1 for the masked MoE layout: the amax over the valid rows only (row i
// of expert e's slab is valid for i < clamp(counts[e], 0, slab)).
__global__ void amax_rows_kernel(int slab, int K, size_t n8, const uint16_t *__restrict__ x,
                                 const int32_t *__restrict__ counts, unsigned int *__restrict__ amax_bits) {
  const size_t row8 = (size_t)K / 8;
  float a = 0.f;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const size_t row = i / row8;
    const int e = (int)(row / slab), r = (int)(row % slab);
    const int c = min(max(counts[e], 0), slab);
    if (r >= c) continue;
    const uint4 v = reinterpret_cast<const uint4 *>(x)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) a = fmaxf(a, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0 && a > 0.f) atomicMax(amax_bits, __float_as_uint(a));
}

__device__ __forceinline__ float nvfp4_global(const unsigned int *amax_bits, const float *static_global) {
  if (static_global) return *static_global;
  const float amax = __uint_as_float(*amax_bits);
  return (amax == 0.f) ? 1.f : __fdiv_rn(amax, 2688.f);
}

// Pass 2: one thread per 16-element block.
__global__ void quant_nvfp4_kernel(size_t nblocks, const uint16_t *__restrict__ x, uint8_t *__restrict__ q,
                                   uint8_t *__restrict__ scales, const unsigned int *__restrict__ amax_bits,
                                   const float *__restrict__ static_global, float *__restrict__ global_out) {
  const float g = nvfp4_global(amax_bits, static_global);
  if (blockIdx.x == 0 && threadIdx.x == 0 && global_out) *global_out = g;
  for (size_t b = blockIdx.x * (size_t)blockDim.x + threadIdx.x; b < nblocks; b += (size_t)gridDim.x * blockDim.x) {
    const uint4 *src = reinterpret_cast<const uint4 *>(x + b * 16);
    uint32_t w[8];
    const uint4 v0 = src[0], v1 = src[1];
    w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
    w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
    const float sbv = __fdiv_rn(__fdiv_rn(amax, 6.f), g);
    const uint32_t sb = f32x2_to_e4m3x2(sbv, 0.f) & 0xFFu;
    scales[b] = (uint8_t)sb;
    const float d = __fmul_rn(e4m3_to_f32(sb), g);
    uint32_t o0 = 0, o1 = 0;
    if (d != 0.f) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o0 |= f32x2_to_e2m1x2(__fdiv_rn(bf16_lo(w[i]), d), __fdiv_rn(bf16_hi(w[i]), d)) << (8 * i);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o1 |= f32x2_to_e2m1x2(__fdiv_rn(bf16_lo(w[4 + i]), d), __fdiv_rn(bf16_hi(w[4 + i]), d)) << (8 * i);
    }
    reinterpret_cast<uint2 *>(q)[b] = make_uint2(o0, o1);
  }
}

// ---- exact decode of quantised activations to bf16 -------------------------
// out[r] = decode(row src(r)) with src(r) = idx ? idx[r] / div : r.
// FP8 per token: the E4M3 value (the per-token scale stays with the GEMM
// epilogue); MXFP8: e4m3 * 2^(c-127); NVFP4: e2m1 * ue4m3 (the global scale
// stays with the epilogue).  All products are exact in fp32 and in bf16
// (at most 4 and 6 significant bits).
__global__ void act_decode_kernel(int afmt, int R, int K, const uint8_t *__restrict__ codes,
                                  const uint8_t *__restrict__ scales, const int32_t *__restrict__ idx, int div,
                                  uint16_t *__restrict__ out) {
  const int per_row = K / 16;  // 16-element chunks
  const size_t total = (size_t)R * per_row;
  for (size_t c = blockIdx.x * (size_t)blockDim.x + threadIdx.x; c < total; c += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(c / per_row), ch = (int)(c % per_row);
    const int src = idx ? idx[r] / div : r;
    const int k0 = ch * 16;
    float v[16];
    if (afmt == A_NVFP4) {
      const uint2 cw = reinterpret_cast<const uint2 *>(codes + (size_t)src * (K / 2))[ch];
      const float s = e4m3_to_f32(scales[(size_t)src * (K / 16) + ch]);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = e2m1_to_f32((cw.x >> (4 * i)) & 15u) * s;
#pragma unroll
      for (int i = 0; i < 8; ++i) v[8 + i] = e2m1_to_f32((cw.y >> (4 * i)) & 15u) * s;
    } else {
      const uint4 cw = reinterpret_cast<const uint4 *>(codes + (size_t)src * K)[ch];
      const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
      float s = 1.f;
      if (afmt == A_MXFP8) s = exp2i((int)scales[(size_t)src * (K / 32) + k0 / 32] - 127);
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = e4m3_to_f32((w[i >> 2] >> (8 * (i & 3))) & 0xFFu) * s;
    }
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i]));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(v[2 * i + 1]));
      o[i] = lo | (hi << 16);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(out + (size_t)r * K + k0);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// ---- bf16 row gather (MoE grouped mode) ------------------------------------
__global__ void gather_rows_kernel(int R, int K, const uint16_t *__restrict__ a, const int32_t *__restrict__ idx,
                                   int div, uint16_t *__restrict__ out) {
  const int per_row = K / 8;
  const size_t total = (size_t)R * per_row;
  for (size_t c = blockIdx.x * (size_t)blockDim.x + threadIdx.x; c < total; c += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(c / per_row), ch = (int)(c % per_row);
    const int src = idx[r] / div;
    reinterpret_cast<uint4 *>(out + (size_t)r * K)[ch] = reinterpret_cast<const uint4 *>(a + (size_t)src * K)[ch];
  }
}

// Row gather of raw bytes (quantised codes or scales): out row r = a row
// idx[r] / div; row_bytes is a multiple of 4.
__global__ void gather_bytes_kernel(int R, int row_bytes, const uint8_t *__restrict__ a,
                                    const int32_t *__restrict__ idx, int div, uint8_t *__restrict__ out) {
  const int per_row = row_bytes / 4;
  const size_t total = (size_t)R * per_row;
  for (size_t c = blockIdx.x * (size_t)blockDim.x + threadIdx.x; c < total; c += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(c / per_row), ch = (int)(c % per_row);
    const int src = idx[r] / div;
    reinterpret_cast<uint32_t *>(out + (size_t)r * row_bytes)[ch] =
        reinterpret_cast<const uint32_t *>(a + (size_t)src * row_bytes)[ch];
  }
}

static int quant_grid(size_t total, int threads) {
  size_t b = (total + threads - 1) / threads;
  if (b > 148 * 16) b = 148 * 16;
  if (b < 1) b = 1;
  return (int)b;
}

hq_status launch_quant_act(int afmt, int M, int K, const void *x, void *codes, void *scales, float *global_out,
                           const float *static_global, void *workspace, cudaStream_t st) {
  if (M == 0) return HQ_OK;
  const uint16_t *xb = (const uint16_t *)x;
  switch (afmt) {
    case A_FP8:
      quant_fp8_token_kernel<<<M, 256, 0, st>>>(M, K, xb, (uint8_t *)codes, (float *)scales);
      break;
    case A_FP8G: {
      const size_t ng = (size_t)M * K / 128;
      quant_fp8_group_kernel<<<quant_grid(ng * 32, 256), 256, 0, st>>>(ng, xb, (uint8_t *)codes, (float *)scales);
      break;
    }
    case A_MXFP8: {
      const size_t nb = (size_t)M * K / 32;
      quant_mxfp8_kernel<<<quant_grid(nb, 128), 128, 0, st>>>(nb, xb, (uint8_t *)codes, (uint8_t *)scales);
      break;
    }
    case A_NVFP4: {
      unsigned int *amax = (unsigned int *)workspace;
      if (!static_global) {
        if (cudaMemsetAsync(amax, 0, sizeof(unsigned int), st) != cudaSuccess) return HQ_ERR_CUDA;
        const size_t n8 = (size_t)M * K / 8;
        amax_kernel<<<quant_grid(n8, 256), 256, 0, st>>>(n8, xb, amax);
      }
      const size_t nb = (size_t)M * K / 16;
      quant_nvfp4_kernel<<<quant_grid(nb, 128), 128, 0, st>>>(nb, xb, (uint8_t *)codes, (uint8_t *)scales, amax,
                                                           static_global, global_out);
      break;
    }
    default:
      return HQ_ERR_UNSUPPORTED;
  }
  return check_launch();
}


// Quantisation of a masked MoE block [E * slab, K]: every row is quantised
// (the rows past an expert's count are never read by the GEMM), but the NVFP4
// tensor scale comes from the valid rows alone, so that it is the one the
// valid rows would get on their own.
hq_status launch_quant_act_masked(int afmt, int E, int slab, int K, const void *x, const int32_t *counts,
                                  void *codes, void *scales, float *global_out, void *workspace, cudaStream_t st) {
  const int M = E * slab;
  if (afmt != A_NVFP4) return launch_quant_act(afmt, M, K, x, codes, scales, global_out, nullptr, workspace, st);
  const uint16_t *xb = (const uint16_t *)x;
  unsigned int *amax = (unsigned int *)workspace;
  if (cudaMemsetAsync(amax, 0, sizeof(unsigned int), st) != cudaSuccess) return HQ_ERR_CUDA;
  const size_t n8 = (size_t)M * K / 8;
  amax_rows_kernel<<<quant_grid(n8, 256), 256, 0, st>>>(slab, K, n8, xb, counts, amax);
  const size_t nb = (size_t)M * K / 16;
  quant_nvfp4_kernel<<<quant_grid(nb, 128), 128, 0, st>>>(nb, xb, (uint8_t *)codes, (uint8_t *)scales, amax,
                                                       nullptr, global_out);
  return check_launch();
}

hq_status launch_act_decode(int afmt, int R, int K, const void *codes, const void *scales, const int32_t *idx,
                            int div, void *out, cudaStream_t st) {
  if (R == 0) return HQ_OK;
  const size_t n = (size_t)R * (K / 16);
  act_decode_kernel<<<quant_grid(n, 256), 256, 0, st>>>(afmt, R, K, (const uint8_t *)codes, (const uint8_t *)scales,
                                                       idx, div, (uint16_t *)out);
  return check_launch();
}

hq_status launch_gather_rows(int R, int K, const void *a, const int32_t *idx, int div, void *out, cudaStream_t st) {
  if (R == 0) return HQ_OK;
  const size_t n = (size_t)R * (K / 8);
  gather_rows_kernel<<<quant_grid(n, 256), 256, 0, st>>>(R, K, (const uint16_t *)a, idx, div, (uint16_t *)out);
  return check_launch();
}

hq_status launch_gather_bytes(int R, int row_bytes, const void *a, const int32_t *idx, int div, void *out,
                              cudaStream_t st) {
  if (R == 0) return HQ_OK;
  if (row_bytes % 4) return HQ_ERR_INVALID_ARG;
  const size_t n = (size_t)R * (row_bytes / 4);
  gather_bytes_kernel<<<quant_grid(n, 256), 256, 0, st>>>(R, row_bytes, (const uint8_t *)a, idx, div,
                                                           (uint8_t *)out);
  return check_launch();
}

}  // namespace hq
