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
  if (fmt == W_MXFP4 || fmt == W_NVFP4 || fmt == W_E0M3) {
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
        v = std_code(L.fmt, ce, L.K, L.std_row(r), k);
        if (L.fmt == W_INT4 || L.fmt == W_MXINT4) v ^= 8u;  // two's complement -> biased (q + 8)
        // float4e0m3 (sign, magnitude m) is the symmetric integer +-m: biased 8 +- m
        if (L.fmt == W_E0M3) v = (v & 8u) ? 8u - (v & 7u) : 8u + v;
      } else if (L.fmt == W_INT4 || L.fmt == W_MXINT4 || L.fmt == W_E0M3) {
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
    const int sr = L.std_row(r);  // standard-format row of packed row r
    if (L.fmt == W_FP8) {
      if (gi == 0) {
        float c = 0.f;
        if (r < L.N) c = reinterpret_cast<const float *>(scales)[(size_t)e * L.N + sr];
        reinterpret_cast<float *>(base + L.c_off)[(size_t)nt * TILE_N + i] = c;
      }
    } else if (L.sbytes == 2) {
      uint16_t s = 0;
      if (r < L.N) s = reinterpret_cast<const uint16_t *>(scales)[((size_t)e * L.N + sr) * L.G + gi];
      reinterpret_cast<uint16_t *>(base + L.s_off)[dst] = s;
    } else {
      uint8_t s = 0;
      if (r < L.N) s = scales[((size_t)e * L.N + sr) * L.G + gi];
      (base + L.s_off)[dst] = s;
    }
    if (L.fmt == W_UINT4) {
      uint8_t z = 0;
      if (r < L.N) {
        const int zw = (L.G + 7) / 8;
        const uint32_t w = reinterpret_cast<const uint32_t *>(zeros)[((size_t)e * L.N + sr) * zw + gi / 8];
        z = (uint8_t)((w >> (4 * (gi % 8))) & 15u);
      }
      (base + L.z_off)[dst] = z;
    } else if (L.fmt == W_UINT1 || L.fmt == W_UINT2 || L.fmt == W_UINT3) {
      (base + L.z_off)[dst] = (r < L.N) ? zeros[((size_t)e * L.N + sr) * L.G + gi] : (uint8_t)0;
    }
    if (L.fmt == W_NVFP4 && r == 0 && gi == 0) {
      reinterpret_cast<float *>(base + L.g_off)[0] = global_scale[e];
    }
  }
}

// Inverse: one thread per standard-format code word/byte.
__global__ void unpack_codes_kernel(Layout L, int E, const uint8_t *packed, uint8_t *codes) {
  // elements per standard-format storage unit
  const int per = (L.fmt == W_FP8) ? 1 : (L.fmt == W_MXFP4 || L.fmt == W_NVFP4 || L.fmt == W_E0M3) ? 2 : 8;
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
    const int pr = L.packed_row(r);
    const int nt = pr / TILE_N, i_row = pr % TILE_N;
    uint32_t out = 0;
    for (int j = 0; j < per; ++j) {
      const int k = u * per + j;
      const int kb = k / TILE_K, kk = k % TILE_K;
      const FragPos fp = frag_pos(L.wbits, i_row, kk);
      const size_t unit = (size_t)nt * L.KB + kb;
      uint32_t v = (pw[unit * words_per_unit + fp.word] >> fp.shift) & ((1u << L.wbits) - 1u);
      if (L.fmt == W_INT4 || L.fmt == W_MXINT4) v ^= 8u;
      if (L.fmt == W_E0M3) v = v >= 8u ? v - 8u : (8u | (8u - v));  // back to sign and magnitude (0 is +0)
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
    const int pr = L.packed_row(r);
    const int nt = pr / TILE_N, i = pr % TILE_N;
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
    if ((L.fmt == W_UINT1 || L.fmt == W_UINT2 || L.fmt == W_UINT3)) zeros[((size_t)e * L.N + r) * L.G + gi] = (base + L.z_off)[src];
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
    if (r < L.N) v = reinterpret_cast<const uint4 *>(codes + ((size_t)e * L.N + L.std_row(r)) * rb)[c];
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
          (r < L.N) ? reinterpret_cast<const float *>(scales)[(size_t)e * L.N + L.std_row(r)] : 0.f;
      continue;
    }
    if (L.bs == BS_F8B) {
      // one fp32 scale per (128-row tile, 128 k): standard [E][NT][K / 128]
      if (i == 0)
        reinterpret_cast<float *>(base + L.c_off)[(size_t)nt * L.G + gi] =
            reinterpret_cast<const float *>(scales)[((size_t)e * L.NT + nt) * L.G + gi];
      continue;
    }
    const uint8_t sv = (r < L.N) ? scales[((size_t)e * L.N + L.std_row(r)) * L.G + gi] : (uint8_t)0;
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
          packed + (size_t)e * L.stride + L.w_off + L.bs_chunk_off(L.packed_row(r), (int)(c * 16 / cb)) +
          (c * 16) % cb);
    } else {
      const size_t j = idx - total_c;
      const int e = (int)(j / ((size_t)L.N * L.G));
      const int rem = (int)(j % ((size_t)L.N * L.G));
      const int r = rem / L.G, gi = rem % L.G;
      const int pr = L.packed_row(r);
      const int nt = pr / TILE_N, i = pr % TILE_N;
      const uint8_t *base = packed + (size_t)e * L.stride;
      if (L.bs == BS_F8) {
        reinterpret_cast<float *>(scales)[(size_t)e * L.N + r] = reinterpret_cast<const float *>(base + L.c_off)[pr];
        continue;
      }
      if (L.bs == BS_F8B) {
        if ((r % TILE_N) == 0)
          reinterpret_cast<float *>(scales)[((size_t)e * L.NT + r / TILE_N) * L.G + gi] =
              reinterpret_cast<const float *>(base + L.c_off)[(size_t)(r / TILE_N) * L.G + gi];
        continue;
      }
      scales[j] = base[L.s_off + ((size_t)nt * (L.G / 4) + gi / 4) * 512 + bs_sf_offset(i, gi & 3)];
      if (L.fmt == W_NVFP4 && r == 0 && gi == 0) global_scale[e] = reinterpret_cast<const float *>(base + L.g_off)[0];
    }
  }
}

// ---- low-bit layouts (2-, 3- and 6-bit codes) ---------------------------------------
// Code k of row r of a b-bit little-endian code stream (row_bytes per row).
__device__ inline uint32_t stream_code(const uint8_t *codes, size_t row_bytes, int r, int k, int b) {
  const uint8_t *row = codes + (size_t)r * row_bytes;
  const int bit = b * k, byte = bit >> 3, off = bit & 7;
  uint32_t v = row[byte];
  if (off + b > 8) v |= (uint32_t)row[byte + 1] << 8;
  return (v >> off) & ((1u << b) - 1u);
}

// Signed codes are stored biased (two's complement -> + 2^(b-1)), so every
// integer format decodes as (u - z).
__device__ inline bool lowbit_signed(int fmt) { return fmt == W_INT1 || fmt == W_INT2 || fmt == W_INT3; }

// The stored (biased) code of packed row p (of the tile order), k of the
// matrix; padded rows decode to zero.
__device__ inline uint32_t lowbit_stored(const Layout &L, const uint8_t *ce, size_t rb, int p, int k) {
  const int b = L.wbits;
  if (p >= L.N) return lowbit_signed(L.fmt) ? (1u << (b - 1)) : 0u;
  uint32_t c = stream_code(ce, rb, L.std_row(p), k, b);
  if (lowbit_signed(L.fmt)) c ^= 1u << (b - 1);
  return c;
}

// One thread per packed 32-bit word of the planes (see plane2_off /
// plane1_off in hq_internal.cuh).
__global__ void pack_lowbit_kernel(Layout L, int E, const uint8_t *codes, uint8_t *packed) {
  const int b = L.wbits;
  const size_t rb = (size_t)L.K * b / 8;
  const size_t wpu = L.unit_bytes() / 4;
  const int p4w = (b == 6) ? 1024 : 0;  // words of the 4-bit plane
  const int p2w = (b == 1) ? 0 : 512;   // words of the 2-bit plane
  const size_t total = (size_t)E * L.NT * L.KB * wpu;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / ((size_t)L.NT * L.KB * wpu));
    const size_t rem = idx % ((size_t)L.NT * L.KB * wpu);
    const size_t unit = rem / wpu;
    const int wi = (int)(rem % wpu);
    const int nt = (int)(unit / L.KB), kb = (int)(unit % L.KB);
    const uint8_t *ce = codes + (size_t)e * L.N * rb;
    uint32_t word = 0;
    if (wi < p4w) {
      // low nibbles of 6-bit codes, in the INT4 unit order
      const int chunk = wi / (TILE_N * 4), i_row = (wi / 4) % TILE_N, j = wi % 4;
      for (int slot = 0; slot < 8; ++slot) {
        const int kk = chunk * 32 + j * 8 + 2 * (slot & 3) + (slot >> 2);
        word |= (lowbit_stored(L, ce, rb, nt * TILE_N + i_row, kb * TILE_K + kk) & 15u) << (4 * slot);
      }
    } else if (wi < p4w + p2w) {
      // 2-bit plane: low two bits (2-, 3-bit codes) or high two (6-bit)
      const int w = wi - p4w, i_row = w / 4, j = w % 4;
      const int sh = (b == 6) ? 4 : 0;
      for (int p = 0; p < 16; ++p) {
        const int kk = 16 * j + (p < 8 ? 2 * p : 2 * (p - 8) + 1);
        word |= ((lowbit_stored(L, ce, rb, nt * TILE_N + i_row, kb * TILE_K + kk) >> sh) & 3u) << (2 * p);
      }
    } else {
      // 1-bit plane: the high bit of 3-bit codes, or 1-bit codes
      const int w = wi - p4w - p2w, i_row = w / 2, j = w % 2;
      const int sh = (b == 3) ? 2 : 0;
      for (int p = 0; p < 32; ++p) {
        const int kk = 32 * j + (p < 16 ? 2 * p : 2 * (p - 16) + 1);
        word |= ((lowbit_stored(L, ce, rb, nt * TILE_N + i_row, kb * TILE_K + kk) >> sh) & 1u) << p;
      }
    }
    reinterpret_cast<uint32_t *>(packed + (size_t)e * L.stride + L.w_off)[unit * wpu + wi] = word;
  }
}

// Inverse: one thread per 8 codes of a standard row (b bytes of the stream).
__global__ void unpack_lowbit_kernel(Layout L, int E, const uint8_t *packed, uint8_t *codes) {
  const int b = L.wbits;
  const size_t rb = (size_t)L.K * b / 8;
  const size_t wpu = L.unit_bytes() / 4;
  const int p4w = (b == 6) ? 1024 : 0;
  const int p2w = (b == 1) ? 0 : 512;
  const size_t per_row = (size_t)L.K / 8;
  const size_t total = (size_t)E * L.N * per_row;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / ((size_t)L.N * per_row));
    const size_t rem = idx % ((size_t)L.N * per_row);
    const int r = (int)(rem / per_row), g8 = (int)(rem % per_row);
    const int pr = L.packed_row(r);
    const int nt = pr / TILE_N, i_row = pr % TILE_N;
    const uint32_t *pw = reinterpret_cast<const uint32_t *>(packed + (size_t)e * L.stride + L.w_off);
    uint64_t bitsacc = 0;
    for (int q = 0; q < 8; ++q) {
      const int k = g8 * 8 + q, kb = k / TILE_K, kk = k % TILE_K;
      const uint32_t *u = pw + ((size_t)nt * L.KB + kb) * wpu;
      uint32_t c = 0;
      if (b == 6) {
        const int ko = kk & 7, slot = (ko & 1) * 4 + (ko >> 1);
        c = (u[((kk >> 5) * TILE_N + i_row) * 4 + ((kk & 31) >> 3)] >> (4 * slot)) & 15u;
      }
      if (b != 1) {
        const int ko = kk & 15, p = (ko & 1) ? 8 + (ko >> 1) : (ko >> 1);
        const uint32_t f = (u[p4w + i_row * 4 + (kk >> 4)] >> (2 * p)) & 3u;
        c |= (b == 6) ? (f << 4) : f;
      }
      if (b == 3 || b == 1) {
        const int ko = kk & 31, p = (ko & 1) ? 16 + (ko >> 1) : (ko >> 1);
        c |= ((u[p4w + p2w + i_row * 2 + (kk >> 5)] >> p) & 1u) << (b == 3 ? 2 : 0);
      }
      if (lowbit_signed(L.fmt)) c ^= 1u << (b - 1);
      bitsacc |= (uint64_t)c << (b * q);
    }
    uint8_t *dst = codes + ((size_t)e * L.N + r) * rb + (size_t)g8 * b;
    for (int i = 0; i < b; ++i) dst[i] = (uint8_t)(bitsacc >> (8 * i));
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
  if (fmt_lowbit(L.fmt))
    pack_lowbit_kernel<<<pack_grid(words, 256), 256, 0, st>>>(L, E, (const uint8_t *)codes, (uint8_t *)packed);
  else
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
  if (fmt_lowbit(L.fmt)) {
    const size_t n8 = (size_t)E * L.N * (L.K / 8);
    unpack_lowbit_kernel<<<pack_grid(n8, 256), 256, 0, st>>>(L, E, (const uint8_t *)packed, (uint8_t *)codes);
  } else {
    const int per = (L.fmt == W_FP8) ? 1 : (L.fmt == W_MXFP4 || L.fmt == W_NVFP4 || L.fmt == W_E0M3) ? 2 : 8;
    const size_t n = (size_t)E * L.N * (L.K / per);
    unpack_codes_kernel<<<pack_grid(n, 256), 256, 0, st>>>(L, E, (const uint8_t *)packed, (uint8_t *)codes);
  }
  const size_t side = (size_t)E * L.N * L.G;
  unpack_side_kernel<<<pack_grid(side, 256), 256, 0, st>>>(L, E, (const uint8_t *)packed, (uint8_t *)scales,
                                                          (uint8_t *)zeros, global_scale);
  return check_launch();
}

}  // namespace hq
