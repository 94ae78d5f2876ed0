// Weight repack: standard format -> MMA-fragment-ordered tiles, and back.
// ("Announcing Humming", section "Tuning & JIT per workload": parameters are
// validated, dimensions padded and tensors repacked into the layout of the
// target kernel.)  The layout is documented in hq_internal.cuh.
#include "hq_internal.cuh"

namespace hq {

// Position of the (row, k) element inside a 64x64 unit:
//   word index inside the unit (32-bit words) and bit offset inside the word.
struct FragPos {
  uint32_t word;
  uint32_t shift;
};

__host__ __device__ inline FragPos frag_pos(int wbits, int i_row, int kk) {
  const int p = i_row >> 4, rr = i_row & 15;
  const int g = rr & 7, hi_row = rr >> 3;
  const int s = kk >> 4, c = kk & 15;
  const int hi_k = c >> 3, c8 = c & 7;
  const int t = c8 >> 1, odd = c8 & 1;
  const int lane = g * 4 + t;
  const int e = (hi_k ? 4 : 0) + (hi_row ? 2 : 0) + odd;  // fragment element 0..7
  FragPos fp;
  if (wbits == 4) {
    fp.word = (uint32_t)((p * 32 + lane) * 4 + s);
    fp.shift = (uint32_t)(4 * ((e >> 1) + 4 * (e & 1)));
  } else {
    const int ew = e & 3;  // element inside its word
    fp.word = (uint32_t)(p * 256 + (s >> 1) * 128 + lane * 4 + 2 * (s & 1) + (e >> 2));
    fp.shift = (uint32_t)(8 * (((ew & 1) << 1) | (ew >> 1)));
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
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(idx / words_per_expert);
    const size_t rem = idx % words_per_expert;
    const size_t unit = rem / words_per_unit;
    const uint32_t wi = (uint32_t)(rem % words_per_unit);
    const int nt = (int)(unit / L.KB), kb = (int)(unit % L.KB);
    const size_t code_stride = (L.fmt == W_FP8) ? (size_t)L.N * L.K
                               : (L.fmt == W_MXFP4 || L.fmt == W_NVFP4) ? (size_t)L.N * L.K / 2
                                                                        : (size_t)L.N * L.K / 2;
    const uint8_t *ce = codes + (size_t)e * code_stride;
    uint32_t word = 0;
    const int per = 32 / L.wbits;
    // enumerate the elements of this word by scanning the unit's 64x64
    // positions that map here: invert frag_pos directly
    for (int slot = 0; slot < per; ++slot) {
      // decode (row, kk) from (wi, slot)
      int i_row, kk;
      if (L.wbits == 4) {
        const int p = wi / 128, lane = (wi / 4) % 32, s = wi % 4;
        const int pos = slot;                       // nibble position
        const int e_el = ((pos & 3) << 1) | (pos >> 2);  // inverse of (e>>1)+4*(e&1)
        const int g = lane / 4, t = lane % 4;
        const int hi_k = e_el >> 2, hi_row = (e_el >> 1) & 1, odd = e_el & 1;
        i_row = p * 16 + hi_row * 8 + g;
        kk = s * 16 + hi_k * 8 + t * 2 + odd;
      } else {
        const int p = wi / 256, h = (wi / 128) % 2, lane = (wi / 4) % 32, w4 = wi % 4;
        const int s = 2 * h + (w4 >> 1), which = w4 & 1;
        const int bpos = slot;                           // byte position in word
        const int ew = ((bpos & 1) << 1) | (bpos >> 1);  // inverse of byte order [e0 e2 e1 e3]
        const int e_el = which * 4 + ew;
        const int g = lane / 4, t = lane % 4;
        const int hi_k = e_el >> 2, hi_row = (e_el >> 1) & 1, odd = e_el & 1;
        i_row = p * 16 + hi_row * 8 + g;
        kk = s * 16 + hi_k * 8 + t * 2 + odd;
      }
      const int r = nt * TILE_N + i_row;
      const int k = kb * TILE_K + kk;
      uint32_t v = 0;
      if (r < L.N) {
        v = std_code(L.fmt, ce, L.K, r, k);
        if (L.fmt == W_INT4) v ^= 8u;  // two's complement -> biased (q + 8)
      } else if (L.fmt == W_INT4) {
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
      if (L.fmt == W_INT4) v ^= 8u;
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

static int pack_grid(size_t total, int threads) {
  size_t b = (total + threads - 1) / threads;
  if (b > 148 * 64) b = 148 * 64;
  if (b < 1) b = 1;
  return (int)b;
}

hq_status launch_pack(const Layout &L, int E, const void *codes, const void *scales, const void *zeros,
                      const float *global_scale, void *packed, cudaStream_t st) {
  const size_t words = (size_t)E * L.NT * L.KB * (L.unit_bytes() / 4);
  pack_weights_kernel<<<pack_grid(words, 256), 256, 0, st>>>(L, E, (const uint8_t *)codes, (uint8_t *)packed);
  const size_t side = (size_t)E * L.NT * TILE_N * L.G;
  pack_side_kernel<<<pack_grid(side, 256), 256, 0, st>>>(L, E, (const uint8_t *)scales, (const uint8_t *)zeros,
                                                        global_scale, (uint8_t *)packed);
  return check_launch();
}

hq_status launch_unpack(const Layout &L, int E, const void *packed, void *codes, void *scales, void *zeros,
                        float *global_scale, cudaStream_t st) {
  const int per = (L.fmt == W_FP8) ? 1 : (L.fmt == W_MXFP4 || L.fmt == W_NVFP4) ? 2 : 8;
  const size_t n = (size_t)E * L.N * (L.K / per);
  unpack_codes_kernel<<<pack_grid(n, 256), 256, 0, st>>>(L, E, (const uint8_t *)packed, (uint8_t *)codes);
  const size_t side = (size_t)E * L.N * L.G;
  unpack_side_kernel<<<pack_grid(side, 256), 256, 0, st>>>(L, E, (const uint8_t *)packed, (uint8_t *)scales,
                                                          (uint8_t *)zeros, global_scale);
  return check_launch();
}

}  // namespace hq
