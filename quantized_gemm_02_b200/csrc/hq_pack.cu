// Weight repack: standard format -> MMA-fragment-ordered tiles, and back.
// ("Announcing Humming", section "Tuning & JIT per workload": parameters are
// validated, dimensions padded and tensors repacked into the layout of the
// target kernel.)  The layout is documented in hq_internal.cuh.
#include "hq_internal.cuh"

namespace hq {

// Position of element (row i_row, k offset kk) inside one 128 x 64 unit:
// 32-bit word index inside the unit and bit offset inside the word.
struct FragPos {
  uint32_t word;
  uint32_t shift;
};

__host__ __device__ inline FragPos frag_pos(int wbits, int i_row, int kk) {
  FragPos fp;
  if (wbits == 4) {
    const int chunk = kk >> 5, kc = kk & 31, j = kc >> 3, ko = kc & 7;
    const int pos = (ko & 1) * 4 + (ko >> 1);  // nibble holding k offset ko
    fp.word = (uint32_t)((chunk * TILE_N + i_row) * 4 + j);
    fp.shift = (uint32_t)(4 * pos);
  } else {
    const int chunk = kk >> 4, kc = kk & 15, j = kc >> 2, ko = kc & 3;
    const int pos = (ko & 1) * 2 + (ko >> 1);  // byte holding k offset ko
    fp.word = (uint32_t)((chunk * TILE_N + i_row) * 4 + j);
    fp.shift = (uint32_t)(8 * pos);
  }
  return fp;
}

// Raw code (nibble or byte) of the standard-format element (r, k).
__device__ inline uint32_t std_code(int fmt, const uint8_t *codes, int K, int r, int k) {
  if (fmt == W_FP8) return codes[(size_t)r * K + k];
  if (fmt == W_MXFP4 || fmt == W_NVFP4) {
    const uint8_t b = codes[(size_t)r * (K / 2) + (k >> 1)];
    return (k & 1) ? (b >> 4) : (b & 15);
  }
  const uint32_t w = reinterpret_cast<const uint32_t *>(codes)[(size_t)r * (K / 8) + (k >> 3)];
  return (w >> (4 * (k & 7))) & 15u;
}

// One thread per packed 32-bit weight word.
__global__ void pack_weights_kernel(Layout L, int E, const uint8_t *codes, uint8_t *packed) {
  const size_t words_per_unit = L.unit_bytes() / 4;
  const size_t words_per_expert = (size_t)L.NT * L.KB * words_per_unit;
  const size_t total = words_per_expert * E;
  const size_t code_stride = (L.fmt == W_FP8) ? (size_t)L.N * L.K : (size_t)L.N * L.K / 2;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / words_per_expert);
    const size_t rem = idx % words_per_expert;
    const size_t unit = rem / words_per_unit;
    const uint32_t wi = (uint32_t)(rem % words_per_unit);
    const int nt = (int)(unit / L.KB), kb = (int)(unit % L.KB);
    const uint8_t *ce = codes + (size_t)e * code_stride;
    const int chunk = (int)(wi / (TILE_N * 4)), i_row = (int)((wi / 4) % TILE_N), j = (int)(wi % 4);
    const int r = nt * TILE_N + i_row;
    uint32_t word = 0;
    const int per = 32 / L.wbits;
    for (int slot = 0; slot < per; ++slot) {
      int kk;
      if (L.wbits == 4) kk = chunk * 32 + j * 8 + 2 * (slot & 3) + (slot >> 2);
      else kk = chunk * 16 + j * 4 + 2 * (slot & 1) + (slot >> 1);
      const int k = kb * TILE_K + kk;
      uint32_t v = 0;
      if (r < L.N) {
        v = std_code(L.fmt, ce, L.K, r, k);
        if (L.fmt == W_INT4 || L.fmt == W_MXINT4) v ^= 8u;  // two's complement -> biased (q + 8)
      } else if (L.fmt == W_INT4 || L.fmt == W_MXINT4) {
        v = 8u;  // padded rows decode to zero
      }
      word |= v << (slot * L.wbits);
    }
    reinterpret_cast<uint32_t *>(packed + (size_t)e * L.stride + L.w_off)[unit * words_per_unit + wi] = word;
  }
}

// Scales, zeros, channel scales and global scale.  One thread per (e, row, group).
__global__ void pack_side_kernel(Layout L, int E, const uint8_t *scales, const uint8_t *zeros,
                                 const float *global_scale, uint8_t *packed) {
  const int R = L.NT * TILE_N;
  const size_t total = (size_t)E * R * L.G;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / ((size_t)R * L.G));
    const int rem = (int)(idx % ((size_t)R * L.G));
    const int r = rem / L.G, gi = rem % L.G;
    const int nt = r / TILE_N, i = r % TILE_N;
    uint8_t *base = packed + (size_t)e * L.stride;
    const size_t dst = ((size_t)nt * L.G + gi) * TILE_N + i;
    if (L.fmt == W_FP8) {
      if (gi == 0) {
        float c = 0.f;
        if (r < L.N) c = reinterpret_cast<const float *>(scales)[(size_t)e * L.N + r];
        reinterpret_cast<float *>(base + L.c_off)[(size_t)nt * TILE_N + i] = c;
      }
    } else if (L.sbytes == 2) {
      uint16_t s = 0;
      if (r < L.N) s = reinterpret_cast<const uint16_t *>(scales)[((size_t)e * L.N + r) * L.G + gi];
      reinterpret_cast<uint16_t *>(base + L.s_off)[dst] = s;
    } else {
      uint8_t s = 0;
      if (r < L.N) s = scales[((size_t)e * L.N + r) * L.G + gi];
      (base + L.s_off)[dst] = s;
    }
    if (L.fmt == W_UINT4) {
      uint8_t z = 0;
      if (r < L.N) {
        const int zw = (L.G + 7) / 8;
        const uint32_t w = reinterpret_cast<const uint32_t *>(zeros)[((size_t)e * L.N + r) * zw + gi / 8];
        z = (uint8_t)((w >> (4 * (gi % 8))) & 15u);
      }
      (base + L.z_off)[dst] = z;
    }
    if (L.fmt == W_NVFP4 && r == 0 && gi == 0) {
      reinterpret_cast<float *>(base + L.g_off)[0] = global_scale[e];
    }
  }
}

// Inverse: one thread per standard-format code word/byte.
__global__ void unpack_codes_kernel(Layout L, int E, const uint8_t *packed, uint8_t *codes) {
  // elements per standard-format storage unit
  const int per = (L.fmt == W_FP8) ? 1 : (L.fmt == W_MXFP4 || L.fmt == W_NVFP4) ? 2 : 8;
  const size_t units_per_row = (size_t)L.K / per;
  const size_t total = (size_t)E * L.N * units_per_row;
  const size_t words_per_unit = L.unit_bytes() / 4;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / ((size_t)L.N * units_per_row));
    const size_t rem = idx % ((size_t)L.N * units_per_row);
    const int r = (int)(rem / units_per_row);
    const int u = (int)(rem % units_per_row);
    const uint32_t *pw = reinterpret_cast<const uint32_t *>(packed + (size_t)e * L.stride + L.w_off);
    const int nt = r / TILE_N, i_row = r % TILE_N;
    uint32_t out = 0;
    for (int j = 0; j < per; ++j) {
      const int k = u * per + j;
      const int kb = k / TILE_K, kk = k % TILE_K;
      const FragPos fp = frag_pos(L.wbits, i_row, kk);
      const size_t unit = (size_t)nt * L.KB + kb;
      uint32_t v = (pw[unit * words_per_unit + fp.word] >> fp.shift) & ((1u << L.wbits) - 1u);
      if (L.fmt == W_INT4 || L.fmt == W_MXINT4) v ^= 8u;
      out |= v << (j * L.wbits);
    }
    if (per == 8) reinterpret_cast<uint32_t *>(codes)[idx] = out;
    else codes[idx] = (uint8_t)out;
  }
}

__global__ void unpack_side_kernel(Layout L, int E, const uint8_t *packed, uint8_t *scales, uint8_t *zeros,
                                   float *global_scale) {
  const size_t total = (size_t)E * L.N * L.G;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / ((size_t)L.N * L.G));
    const int rem = (int)(idx % ((size_t)L.N * L.G));
    const int r = rem / L.G, gi = rem % L.G;
    const int nt = r / TILE_N, i = r % TILE_N;
    const uint8_t *base = packed + (size_t)e * L.stride;
    const size_t src = ((size_t)nt * L.G + gi) * TILE_N + i;
    if (L.fmt == W_FP8) {
      if (gi == 0)
        reinterpret_cast<float *>(scales)[(size_t)e * L.N + r] =
            reinterpret_cast<const float *>(base + L.c_off)[(size_t)nt * TILE_N + i];
    } else if (L.sbytes == 2) {
      reinterpret_cast<uint16_t *>(scales)[idx] = reinterpret_cast<const uint16_t *>(base + L.s_off)[src];
    } else {
      scales[idx] = (base + L.s_off)[src];
    }
    if (L.fmt == W_UINT4 && (gi % 8) == 0) {
      const int zw = (L.G + 7) / 8;
      uint32_t w = 0;
      for (int j = 0; j < 8 && gi + j < L.G; ++j)
        w |= (uint32_t)(base + L.z_off)[((size_t)nt * L.G + gi + j) * TILE_N + i] << (4 * j);
      reinterpret_cast<uint32_t *>(zeros)[((size_t)e * L.N + r) * zw + gi / 8] = w;
    }
    if (L.fmt == W_NVFP4 && r == 0 && gi == 0) global_scale[e] = reinterpret_cast<const float *>(base + L.g_off)[0];
  }
}

// ---- block-scaled layouts ----------------------------------------------------------
// Byte offset of scale column j (0..3 inside its chunk) of tile row i in a
// 512-byte scale chunk: the row's 32-row group picks the 4-byte column
// inside the row's 16-byte line, so that one tensor-memory copy of the chunk
// (32 lanes x 16 bytes, replicated to the four lane quadrants) puts the
// scales of rows i, i + 32, i + 64, i + 96 in four consecutive columns.
__host__ __device__ inline uint32_t bs_sf_offset(int i, int j) { return (uint32_t)((i & 31) * 16 + (i >> 5) * 4 + j); }

// Codes: each row's bytes cut into stage chunks, [NT][chunk][128 rows][chunk
// bytes], rows past N zeroed; 16 bytes per thread.
__global__ void pack_bs_codes_kernel(Layout L, int E, const uint8_t *codes, uint8_t *packed) {
  const size_t rb = L.bs_row_bytes();
  const size_t row16 = rb / 16;  // 16-byte pieces per row
  const size_t rows = (size_t)L.NT * TILE_N;
  const size_t total = (size_t)E * rows * row16;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / (rows * row16));
    const size_t rem = idx % (rows * row16);
    const int r = (int)(rem / row16);
    const size_t c = rem % row16;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r < L.N) v = reinterpret_cast<const uint4 *>(codes + ((size_t)e * L.N + r) * rb)[c];
    const int cb = L.bs_chunk_bytes();
    *reinterpret_cast<uint4 *>(packed + (size_t)e * L.stride + L.w_off +
                               L.bs_chunk_off(r, (int)(c * 16 / cb)) + (c * 16) % cb) = v;
  }
}

// Scales into 512-byte chunks (one thread per scale byte) and the global
// scale; FP8: the per-row fp32 scales, zero past N.
__global__ void pack_bs_side_kernel(Layout L, int E, const uint8_t *scales, const float *global_scale,
                                    uint8_t *packed) {
  const int R = L.NT * TILE_N;
  const size_t total = (size_t)E * R * L.G;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / ((size_t)R * L.G));
    const int rem = (int)(idx % ((size_t)R * L.G));
    const int r = rem / L.G, gi = rem % L.G;
    const int nt = r / TILE_N, i = r % TILE_N;
    uint8_t *base = packed + (size_t)e * L.stride;
    if (L.bs == BS_F8) {
      reinterpret_cast<float *>(base + L.c_off)[r] =
          (r < L.N) ? reinterpret_cast<const float *>(scales)[(size_t)e * L.N + r] : 0.f;
      continue;
    }
    const uint8_t sv = (r < L.N) ? scales[((size_t)e * L.N + r) * L.G + gi] : (uint8_t)0;
    base[L.s_off + ((size_t)nt * (L.G / 4) + gi / 4) * 512 + bs_sf_offset(i, gi & 3)] = sv;
    if (L.fmt == W_NVFP4 && r == 0 && gi == 0) reinterpret_cast<float *>(base + L.g_off)[0] = global_scale[e];
  }
}

__global__ void unpack_bs_kernel(Layout L, int E, const uint8_t *packed, uint8_t *codes, uint8_t *scales,
                                 float *global_scale) {
  const size_t rb = L.bs_row_bytes();
  const size_t row16 = rb / 16;
  const size_t total_c = (size_t)E * L.N * row16;
  const size_t total_s = (size_t)E * L.N * L.G;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total_c + total_s;
       idx += (size_t)gridDim.x * blockDim.x) {
    if (idx < total_c) {
      const int e = (int)(idx / ((size_t)L.N * row16));
      const size_t rem = idx % ((size_t)L.N * row16);
      const int r = (int)(rem / row16);
      const size_t c = rem % row16;
      const int cb = L.bs_chunk_bytes();
      reinterpret_cast<uint4 *>(codes + ((size_t)e * L.N + r) * rb)[c] = *reinterpret_cast<const uint4 *>(
          packed + (size_t)e * L.stride + L.w_off + L.bs_chunk_off(r, (int)(c * 16 / cb)) + (c * 16) % cb);
    } else {
      const size_t j = idx - total_c;
      const int e = (int)(j / ((size_t)L.N * L.G));
      const int rem = (int)(j % ((size_t)L.N * L.G));
      const int r = rem / L.G, gi = rem % L.G;
      const int nt = r / TILE_N, i = r % TILE_N;
      const uint8_t *base = packed + (size_t)e * L.stride;
      if (L.bs == BS_F8) {
        reinterpret_cast<float *>(scales)[(size_t)e * L.N + r] = reinterpret_cast<const float *>(base + L.c_off)[r];
        continue;
      }
      scales[j] = base[L.s_off + ((size_t)nt * (L.G / 4) + gi / 4) * 512 + bs_sf_offset(i, gi & 3)];
      if (L.fmt == W_NVFP4 && r == 0 && gi == 0) global_scale[e] = reinterpret_cast<const float *>(base + L.g_off)[0];
    }
  }
}

static int pack_grid(size_t total, int threads) {
  size_t b = (total + threads - 1) / threads;
  if (b > 148 * 64) b = 148 * 64;
  if (b < 1) b = 1;
  return (int)b;
}

hq_status launch_pack(const Layout &L, int E, const void *codes, const void *scales, const void *zeros,
                      const float *global_scale, void *packed, cudaStream_t st) {
  if (L.bs != BS_NONE) {
    const size_t n16 = (size_t)E * L.NT * TILE_N * (L.bs_row_bytes() / 16);
    pack_bs_codes_kernel<<<pack_grid(n16, 256), 256, 0, st>>>(L, E, (const uint8_t *)codes, (uint8_t *)packed);
    const size_t ns = (size_t)E * L.NT * TILE_N * L.G;
    pack_bs_side_kernel<<<pack_grid(ns, 256), 256, 0, st>>>(L, E, (const uint8_t *)scales, global_scale,
                                                             (uint8_t *)packed);
    return check_launch();
  }
  const size_t words = (size_t)E * L.NT * L.KB * (L.unit_bytes() / 4);
  pack_weights_kernel<<<pack_grid(words, 256), 256, 0, st>>>(L, E, (const uint8_t *)codes, (uint8_t *)packed);
  const size_t side = (size_t)E * L.NT * TILE_N * L.G;
  pack_side_kernel<<<pack_grid(side, 256), 256, 0, st>>>(L, E, (const uint8_t *)scales, (const uint8_t *)zeros,
                                                        global_scale, (uint8_t *)packed);
  return check_launch();
}

hq_status launch_unpack(const Layout &L, int E, const void *packed, void *codes, void *scales, void *zeros,
                        float *global_scale, cudaStream_t st) {
  if (L.bs != BS_NONE) {
    const size_t n = (size_t)E * L.N * (L.bs_row_bytes() / 16) + (size_t)E * L.N * L.G;
    unpack_bs_kernel<<<pack_grid(n, 256), 256, 0, st>>>(L, E, (const uint8_t *)packed, (uint8_t *)codes,
                                                         (uint8_t *)scales, global_scale);
    return check_launch();
  }
  const int per = (L.fmt == W_FP8) ? 1 : (L.fmt == W_MXFP4 || L.fmt == W_NVFP4) ? 2 : 8;
  const size_t n = (size_t)E * L.N * (L.K / per);
  unpack_codes_kernel<<<pack_grid(n, 256), 256, 0, st>>>(L, E, (const uint8_t *)packed, (uint8_t *)codes);
  const size_t side = (size_t)E * L.N * L.G;
  unpack_side_kernel<<<pack_grid(side, 256), 256, 0, st>>>(L, E, (const uint8_t *)packed, (uint8_t *)scales,
                                                          (uint8_t *)zeros, global_scale);
  return check_launch();
}

}  // namespace hq
