// MoE routing prepare and the fused weighted top-k sum.
//
// SGLang integration digest (PR #23754): moe_permute_prepare /
// moe_align_block_size compute per-expert counts and the expert-sorted
// permutation; moe_unpermute / moe_fused_mul_sum bring expert outputs back to
// token order and form sum_j w[t, j] * y[t, j].
#include <cuda_bf16.h>

#include "hq_internal.cuh"

namespace hq {

constexpr int PERM_THREADS = 1024;

// One CTA.  Slots s = t * topk + j are placed stably (increasing s inside an
// expert): chunks of 1024 slots are processed in order; inside a chunk the
// rank of a slot among equal experts is (earlier warps' counts) + (its rank
// among matching lanes of its warp).
__global__ void __launch_bounds__(PERM_THREADS) moe_permute_kernel(int n, int E, const int32_t *__restrict__ ids,
                                                                    int32_t *__restrict__ offsets,
                                                                    int32_t *__restrict__ perm,
                                                                    int32_t *__restrict__ inv) {
  extern __shared__ int sh[];
  int *run = sh;                                                // [E] next free position per expert
  int *chunk_tot = sh + E;                                      // [E] slots of each expert in the chunk
  uint16_t *wpre = reinterpret_cast<uint16_t *>(sh + 2 * E);    // [32][E] per-warp counts -> prefixes
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) bad = 0;
  for (int e = tid; e < E; e += PERM_THREADS) run[e] = 0;
  __syncthreads();
  for (int i = tid; i < n; i += PERM_THREADS) {
    const int e = ids[i];
    if (e < 0 || e >= E) bad = 1;
    else atomicAdd(&run[e], 1);
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      set_device_error(HQ_ERR_DEVICE_INDEX);
      offsets[E] = -1;
    }
    return;
  }
  // exclusive scan of the counts (warp 0)
  if (warp == 0) {
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int c = (e < E) ? run[e] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < E) {
        offsets[e] = carry + incl - c;
        run[e] = carry + incl - c;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) offsets[E] = carry;
  }
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int base = 0; base < n; base += PERM_THREADS) {
    for (int x = tid; x < 32 * E; x += PERM_THREADS) wpre[x] = 0;
    __syncthreads();
    const int i = base + tid;
    const bool valid = i < n;
    const int e = valid ? ids[i] : -1;
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & lt);
    if (valid && rank == 0) wpre[warp * E + e] = (uint16_t)__popc(same);
    __syncthreads();
    for (int x = tid; x < E; x += PERM_THREADS) {
      int acc = 0;
      for (int w = 0; w < 32; ++w) {
        const int c = wpre[w * E + x];
        wpre[w * E + x] = (uint16_t)acc;
        acc += c;
      }
      chunk_tot[x] = acc;
    }
    __syncthreads();
    if (valid) {
      const int pos = run[e] + wpre[warp * E + e] + rank;
      perm[pos] = i;
      inv[i] = pos;
    }
    __syncthreads();
    for (int x = tid; x < E; x += PERM_THREADS) run[x] += chunk_tot[x];
    __syncthreads();
  }
}

// out[t, n] = rs * sum_j w[t, j] * y[r(t, j), n]; 8 columns per thread.
__global__ void unpermute_sum_kernel(int T, int topk, int N, const uint16_t *__restrict__ y,
                                     const int32_t *__restrict__ inv, const float *__restrict__ w, float rs,
                                     uint16_t *__restrict__ out) {
  const int per_row = N / 8;
  const size_t total = (size_t)T * per_row;
  for (size_t c = blockIdx.x * (size_t)blockDim.x + threadIdx.x; c < total; c += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(c / per_row), ch = (int)(c % per_row);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int j = 0; j < topk; ++j) {
      const int s = t * topk + j;
      const int r = inv ? inv[s] : s;
      const float wj = w[s];
      const uint4 v = reinterpret_cast<const uint4 *>(y + (size_t)r * N)[ch];
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fmaf_rn(wj, __uint_as_float(u[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(wj, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i] * rs));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i + 1] * rs));
      o[i] = lo | (hi << 16);
    }
    reinterpret_cast<uint4 *>(out + (size_t)t * N)[ch] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

hq_status launch_moe_permute(int T, int topk, int E, const int32_t *ids, int32_t *offsets, int32_t *perm,
                             int32_t *inv, cudaStream_t st) {
  const int n = T * topk;
  const size_t smem = (size_t)2 * E * sizeof(int) + (size_t)32 * E * sizeof(uint16_t);
  // sized once per device for the largest supported E (1024)
  static unsigned configured = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
  if (dev >= 32 || !(configured & (1u << dev))) {
    const int max_smem = 2 * 1024 * (int)sizeof(int) + 32 * 1024 * (int)sizeof(uint16_t);
    if (cudaFuncSetAttribute(moe_permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem) != cudaSuccess)
      return HQ_ERR_CUDA;
    if (dev < 32) configured |= 1u << dev;
  }
  moe_permute_kernel<<<1, PERM_THREADS, smem, st>>>(n, E, ids, offsets, perm, inv);
  return check_launch();
}

// Masked MoE layout (SGLang digest: humming_moe_runner_core_run, gemm type
// "grouped_masked"): expert e owns rows [e * slab, e * slab + c_e) of an
// [E * slab, K] block, c_e = clamp(counts[e], 0, slab).  Writes the grouped
// path's routing for it: offsets [E + 1], the exclusive prefix of c_e, and
// perm[offsets[e] + i] = e * slab + i; the positions past the total get row
// 0 (staged but never multiplied).  One block per expert, each summing the
// counts before its own; E <= 1024.
__global__ void moe_masked_prepare_kernel(int E, int slab, const int32_t *__restrict__ counts,
                                          int32_t *__restrict__ offsets, int32_t *__restrict__ perm) {
  __shared__ int s_base;
  const int e = blockIdx.x;
  if (threadIdx.x < 32) {
    int sum = 0;
    for (int j = threadIdx.x; j < e; j += 32) sum += min(max(counts[j], 0), slab);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (threadIdx.x == 0) s_base = sum;
  }
  __syncthreads();
  const int base = s_base;
  const int c = min(max(counts[e], 0), slab);
  for (int i = threadIdx.x; i < c; i += blockDim.x) perm[base + i] = e * slab + i;
  if (threadIdx.x == 0) {
    offsets[e] = base;
    if (e == E - 1) offsets[E] = base + c;
  }
  if (e == E - 1)
    for (int r = base + c + threadIdx.x; r < E * slab; r += blockDim.x) perm[r] = 0;
}

hq_status launch_moe_masked_prepare(int E, int slab, const int32_t *counts, int32_t *offsets, int32_t *perm,
                                    cudaStream_t st) {
  moe_masked_prepare_kernel<<<E, 256, 0, st>>>(E, slab, counts, offsets, perm);
  return check_launch();
}

// SiLU-and-mul between the gate-up and the down GEMM of an MoE layer:
// out[r, i] = bf16(silu(g) * u), g = y[r, i], u = y[r, I + i], in fp32 with
// silu(g) = g / (1 + exp(-g)) (expf, IEEE division); 8 columns per thread.
__global__ void silu_and_mul_kernel(int R, int I, const uint16_t *__restrict__ y, uint16_t *__restrict__ out) {
  const int per_row = I / 8;
  const size_t total = (size_t)R * per_row;
  for (size_t c = blockIdx.x * (size_t)blockDim.x + threadIdx.x; c < total; c += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(c / per_row), ch = (int)(c % per_row);
    const uint4 gv = reinterpret_cast<const uint4 *>(y + (size_t)r * 2 * I)[ch];
    const uint4 uv = reinterpret_cast<const uint4 *>(y + (size_t)r * 2 * I + I)[ch];
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float res[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float g = __uint_as_float(h ? (gw[i] & 0xFFFF0000u) : (gw[i] << 16));
        const float u = __uint_as_float(h ? (uw[i] & 0xFFFF0000u) : (uw[i] << 16));
        res[h] = __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), u);
      }
      o[i] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(res[0])) |
             ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(res[1])) << 16);
    }
    reinterpret_cast<uint4 *>(out + (size_t)r * I)[ch] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

hq_status launch_silu_and_mul(int R, int I, const void *y, void *out, cudaStream_t st) {
  if (R == 0) return HQ_OK;
  const size_t total = (size_t)R * (I / 8);
  size_t blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  silu_and_mul_kernel<<<(int)blocks, 256, 0, st>>>(R, I, (const uint16_t *)y, (uint16_t *)out);
  return check_launch();
}

hq_status launch_unpermute_sum(int T, int topk, int N, const void *y, const int32_t *inv, const float *w, float rs,
                               void *out, cudaStream_t st) {
  if (T == 0) return HQ_OK;
  const size_t total = (size_t)T * (N / 8);
  size_t blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  unpermute_sum_kernel<<<(int)blocks, 256, 0, st>>>(T, topk, N, (const uint16_t *)y, inv, w, rs, (uint16_t *)out);
  return check_launch();
}

}  // namespace hq
