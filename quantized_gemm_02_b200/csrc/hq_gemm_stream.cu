// Weight-streaming GEMM for small token counts (decode regime), dense and MoE.
//
// "Announcing Humming", section "Tuning & JIT per workload": at small batch a
// multistage asynchronous-copy + MMA pipeline can beat the TMA/UMMA one; the
// dequantisation is fused into the compute ("Shared CUDA components": decode
// of bit width, int/float, scales and zero points inside the kernel); Stream-K
// style work splitting balances the SMs.  Here, on sm_100a:
//
//   * one producer warp streams the packed weights of a 64-row tile (and the
//     matching scales / zero points / bf16 activation rows) into a 4-stage
//     shared-memory ring with 1-D bulk copies (cp.async.bulk) completing on
//     mbarriers; weights carry an L2 evict-first hint (read exactly once);
//   * four consumer warps each take one 64-k block of every stage, load their
//     16-byte fragment words (the packed layout is already in mma.sync
//     A-fragment order), dequantise in registers to bf16 and issue
//     mma.sync m16n8k16 with W as the A operand (swap-AB: weight rows are
//     the MMA M dimension, tokens the N dimension);
//   * the four warps' fp32 partials are reduced through shared memory; with
//     split-K, every split writes an fp32 partial and the last split to
//     arrive (atomic ticket) sums all of them in split order (deterministic)
//     and applies the epilogue.  Partial sums never pass through bf16.
//
// Dequantisation (exact integer / FP decode, one bf16 rounding for INT4
// scales):  INT4/UINT4: (u - z) * s;  E2M1: bit-move into bf16 then * 2^126
// * s (s = 2^(c-127) for E8M0, the UE4M3 value for NVFP4);  E4M3: bit-move *
// 2^120.  FP8 channel scales, per-token activation scales and NVFP4 global
// scales are applied in fp32 in the epilogue.
#include <cuda_bf16.h>

#include "hq_internal.cuh"

namespace hq {

constexpr int S_KB = 4;        // k-blocks per stage (one per consumer warp)
constexpr int NSTAGE = 4;      // ring depth
constexpr int A_PITCH = S_KB * TILE_K * 2 + 16;  // bytes per activation row in a stage (+16: bank skew)
constexpr int CONSUMERS = 4;
constexpr int THREADS = (CONSUMERS + 1) * 32;

struct StreamParams {
  const uint8_t *packed;  // expert 0
  size_t stride;          // bytes per expert
  size_t w_off, s_off, z_off, c_off, g_off;
  int N, K, NT, KB, G, group;
  const uint16_t *a;      // bf16 activations [rows, K]
  const float *row_scale; // per activation row (FP8 per-token) or null
  const float *a_global;  // NVFP4 activation global scale or null
  int M;                  // dense token count
  int moe;                // 0 dense, 1 MoE
  int E;
  const int32_t *offsets; // [E+1]
  const int32_t *perm;    // [T*k]
  int a_indexed;          // MoE: 1 = activation row perm[p] / a_div, 0 = row p
  int a_div;
  uint16_t *out;          // bf16 [rows, N]
  int splits, kb_per_split;
  float *partial;         // [tiles][splits][MT][64]
  int *counters;          // [tiles]
};

template <int WF>
struct WTraits {
  static constexpr int wbits = (WF == W_FP8) ? 8 : 4;
  static constexpr int unit = TILE_N * TILE_K * wbits / 8;  // bytes per (tile, k-block)
  static constexpr int sbytes = (WF == W_INT4 || WF == W_UINT4) ? 2 : 1;
  static constexpr int group_max_per_stage = (WF == W_NVFP4) ? 16 : (WF == W_MXFP4) ? 8 : 8;  // int g>=32
  static constexpr bool has_scales = (WF != W_FP8);
  static constexpr bool has_zero = (WF == W_UINT4);
  static constexpr bool fp4 = (WF == W_MXFP4 || WF == W_NVFP4);
};

template <int WF, int MT>
struct Smem {
  static constexpr int W = S_KB * WTraits<WF>::unit;
  static constexpr int A = MT * A_PITCH;
  static constexpr int S = WTraits<WF>::group_max_per_stage * TILE_N * WTraits<WF>::sbytes;
  static constexpr int Z = WTraits<WF>::has_zero ? WTraits<WF>::group_max_per_stage * TILE_N : 0;
  static constexpr int SB = WTraits<WF>::fp4 ? WTraits<WF>::group_max_per_stage * TILE_N * 2 : 0;  // bf16 scales
  static constexpr int STAGE = (W + A + S + Z + SB + 127) / 128 * 128;
  static constexpr int RED = CONSUMERS * TILE_N * (MT + 1) * 4;
  static constexpr int RING = NSTAGE * STAGE;
  static constexpr int BYTES = (RING > RED ? RING : RED) + 256;
};

// ---- small PTX helpers -----------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&a), *reinterpret_cast<__nv_bfloat162 *>(&b));
  return *reinterpret_cast<uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&a), *reinterpret_cast<__nv_bfloat162 *>(&b));
  return *reinterpret_cast<uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t bcast16(uint32_t h) { return (h & 0xFFFFu) | (h << 16); }

// bf16 bit pattern of an E4M3 / UE4M3 code value (exact: at most 4
// significant bits, exponent range inside bf16's).
__device__ __forceinline__ uint32_t e4m3_code_to_bf16(uint32_t c) {
  const float mag = __uint_as_float((c & 0x7Fu) << 20) * 1.329227995784916e36f;  // 2^120
  return (__float_as_uint(mag) >> 16) | ((c & 0x80u) << 8);
}
// bf16 bit pattern of 2^(c - 127) for an E8M0 code c in [0, 254].
__device__ __forceinline__ uint32_t e8m0_code_to_bf16(uint32_t c) { return c ? (c << 7) : 0x0040u; }

// ---- fragment decoders: one 32-bit packed word -> four bf16x2 registers ----
// lo = multiplier/zero for row g (registers 0 and 2), hi = row g+8 (1 and 3).
__device__ __forceinline__ void dequant_int(uint32_t w, uint32_t zlo, uint32_t zhi, uint32_t slo, uint32_t shi,
                                            uint32_t (&r)[4]) {
  const uint32_t x0 = (w & 0x000F000Fu) | 0x43004300u;
  const uint32_t x1 = ((w >> 4) & 0x000F000Fu) | 0x43004300u;
  const uint32_t x2 = ((w >> 8) & 0x000F000Fu) | 0x43004300u;
  const uint32_t x3 = ((w >> 12) & 0x000F000Fu) | 0x43004300u;
  r[0] = bmul2(bsub2(x0, zlo), slo);
  r[1] = bmul2(bsub2(x1, zhi), shi);
  r[2] = bmul2(bsub2(x2, zlo), slo);
  r[3] = bmul2(bsub2(x3, zhi), shi);
}

__device__ __forceinline__ uint32_t e2m1_pair(uint32_t x) {
  return ((x << 6) & 0x01C001C0u) | ((x << 12) & 0x80008000u);
}
__device__ __forceinline__ void dequant_fp4(uint32_t w, uint32_t slo, uint32_t shi, uint32_t (&r)[4]) {
  const uint32_t k126 = 0x7E807E80u;  // bf16 2^126 in both halves
  r[0] = bmul2(bmul2(e2m1_pair(w), k126), slo);
  r[1] = bmul2(bmul2(e2m1_pair(w >> 4), k126), shi);
  r[2] = bmul2(bmul2(e2m1_pair(w >> 8), k126), slo);
  r[3] = bmul2(bmul2(e2m1_pair(w >> 12), k126), shi);
}

__device__ __forceinline__ uint32_t e4m3_pair(uint32_t x) {  // bytes at bits 0..7 and 16..23
  return ((x & 0x007F007Fu) << 4) | ((x & 0x00800080u) << 8);
}
__device__ __forceinline__ void dequant_fp8(uint32_t wa, uint32_t wb, uint32_t (&r)[4]) {
  const uint32_t k120 = 0x7B807B80u;  // bf16 2^120
  r[0] = bmul2(e4m3_pair(wa), k120);
  r[1] = bmul2(e4m3_pair(wa >> 8), k120);
  r[2] = bmul2(e4m3_pair(wb), k120);
  r[3] = bmul2(e4m3_pair(wb >> 8), k120);
}

// ---- the kernel -------------------------------------------------------------
template <int WF, int MT>
__global__ void __launch_bounds__(THREADS) stream_gemm_kernel(const StreamParams p) {
  using T = WTraits<WF>;
  using SM = Smem<WF, MT>;
  constexpr int NT8 = MT / 8;  // n8 tiles (tokens)
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + SM::BYTES - 256);
  uint64_t *empty = full + NSTAGE;
  __shared__ int s_arow[MT];  // row of the bf16 activation buffer
  __shared__ int s_srow[MT];  // caller's activation row (per-token scale index)
  __shared__ int s_orow[MT];  // output row
  __shared__ int s_info[4];  // expert, valid tokens, is_last

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nt = blockIdx.x % p.NT;
  const int split = blockIdx.x / p.NT;
  const int slot = blockIdx.y;

  // ---- tile -> (expert, rows) ----
  if (warp == 0) {
    int expert = 0, nvalid = 0, base = 0;
    if (!p.moe) {
      base = slot * MT;
      nvalid = min(MT, p.M - base);
    } else {
      if (p.offsets[p.E] < 0) {
        nvalid = 0;
      } else {
        // prefix over experts of ceil(count / MT), found by one warp
        int running = 0, found = -1, tile_in = 0;
        for (int e0 = 0; e0 < p.E && found < 0; e0 += 32) {
          const int e = e0 + lane;
          int tiles = 0;
          if (e < p.E) tiles = (p.offsets[e + 1] - p.offsets[e] + MT - 1) / MT;
          int incl = tiles;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
          }
          const int excl = running + incl - tiles;
          const bool mine = (e < p.E) && slot >= excl && slot < excl + tiles;
          const unsigned ball = __ballot_sync(0xffffffffu, mine);
          if (ball) {
            const int src = __ffs(ball) - 1;
            found = __shfl_sync(0xffffffffu, e, src);
            tile_in = __shfl_sync(0xffffffffu, slot - excl, src);
          }
          running += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (found >= 0) {
          expert = found;
          base = p.offsets[found] + tile_in * MT;
          nvalid = min(MT, p.offsets[found + 1] - base);
        }
      }
    }
    for (int i = lane; i < MT; i += 32) {
      int ar = -1, sr = -1, orow = -1;
      if (i < nvalid) {
        const int pos = base + i;
        if (!p.moe) {
          ar = sr = orow = pos;
        } else {
          const int s = p.perm[pos];
          sr = s / p.a_div;
          ar = p.a_indexed ? sr : pos;
          orow = s;
        }
      }
      s_arow[i] = ar;
      s_srow[i] = sr;
      s_orow[i] = orow;
    }
    if (lane == 0) {
      s_info[0] = expert;
      s_info[1] = nvalid;
    }
  }
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CONSUMERS);
    }
    fence_barrier_init();
  }
  __syncthreads();
  const int expert = s_info[0], nvalid = s_info[1];
  if (nvalid <= 0) return;

  const uint8_t *eb = p.packed + (size_t)expert * p.stride;
  const int kb_begin = split * p.kb_per_split;
  const int kb_end = min(p.KB, kb_begin + p.kb_per_split);
  const int nst = (kb_end - kb_begin + S_KB - 1) / S_KB;

  if (warp == CONSUMERS) {
    // ================= producer =================
    const uint64_t pol = policy_evict_first();
    for (int it = 0; it < nst; ++it) {
      const int stg = it % NSTAGE;
      if (it >= NSTAGE) {
        if (!mbar_wait(&empty[stg], ((it / NSTAGE) - 1) & 1)) break;
      }
      uint8_t *sbase = smem + stg * SM::STAGE;
      const int kb0 = kb_begin + it * S_KB;
      const int nkb = min(S_KB, kb_end - kb0);
      const int g0 = kb0 * TILE_K / p.group;
      const int g1 = ((kb0 + nkb) * TILE_K + p.group - 1) / p.group;
      const uint32_t wbytes = (uint32_t)(nkb * T::unit);
      const uint32_t abytes = (uint32_t)(nkb * TILE_K * 2);
      const uint32_t sbytes = T::has_scales ? (uint32_t)((g1 - g0) * TILE_N * T::sbytes) : 0u;
      const uint32_t zbytes = T::has_zero ? (uint32_t)((g1 - g0) * TILE_N) : 0u;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[stg], wbytes + abytes * nvalid + sbytes + zbytes);
        const uint8_t *wsrc = eb + p.w_off + ((size_t)nt * p.KB + kb0) * T::unit;
        bulk_g2s_stream(sbase, wsrc, wbytes, &full[stg], pol);
        if (T::has_scales)
          bulk_g2s(sbase + SM::W + SM::A, eb + p.s_off + ((size_t)nt * p.G + g0) * TILE_N * T::sbytes, sbytes,
                   &full[stg]);
        if (T::has_zero)
          bulk_g2s(sbase + SM::W + SM::A + SM::S, eb + p.z_off + ((size_t)nt * p.G + g0) * TILE_N, zbytes,
                   &full[stg]);
      }
      __syncwarp();
      for (int i = lane; i < nvalid; i += 32) {
        const uint16_t *src = p.a + (size_t)s_arow[i] * p.K + (size_t)kb0 * TILE_K;
        bulk_g2s(sbase + SM::W + i * A_PITCH, src, abytes, &full[stg]);
      }
    }
  } else {
    // ================= consumers =================
    float acc[4][NT8][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < NT8; ++b)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.f;

    const int g = lane >> 2;
    for (int it = 0; it < nst; ++it) {
      const int stg = it % NSTAGE;
      if (!mbar_wait(&full[stg], (it / NSTAGE) & 1)) break;
      uint8_t *sbase = smem + stg * SM::STAGE;
      const int kb0 = kb_begin + it * S_KB;
      const int nkb = min(S_KB, kb_end - kb0);
      const int g0 = kb0 * TILE_K / p.group;
      const uint8_t *sS = sbase + SM::W + SM::A;
      uint16_t *sSB = reinterpret_cast<uint16_t *>(sbase + SM::W + SM::A + SM::S + SM::Z);
      if constexpr (T::fp4) {
        // convert this stage's FP4 block scales to bf16 multipliers once
        const int g1 = ((kb0 + nkb) * TILE_K + p.group - 1) / p.group;
        const int n = (g1 - g0) * TILE_N;
        for (int i = tid; i < n; i += CONSUMERS * 32)
          sSB[i] = (uint16_t)((WF == W_MXFP4) ? e8m0_code_to_bf16(sS[i]) : e4m3_code_to_bf16(sS[i]));
        asm volatile("bar.sync 1, %0;" ::"n"(CONSUMERS * 32));
      }
      if (warp < nkb) {
        const int kbl = warp;  // local k-block handled by this warp
        const uint8_t *wb = sbase + kbl * T::unit;
        uint4 wv[4][T::wbits / 4];
#pragma unroll
        for (int pn = 0; pn < 4; ++pn)
#pragma unroll
          for (int h = 0; h < T::wbits / 4; ++h)
            wv[pn][h] = *reinterpret_cast<const uint4 *>(wb + pn * (T::wbits == 4 ? 512 : 1024) + h * 512 +
                                                         lane * 16);
        const uint32_t a_base = smem_u32(sbase + SM::W) + kbl * TILE_K * 2;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          // B fragments (activations) for this k16 step
          uint32_t b[NT8][2];
          if constexpr (MT == 8) {
            const int row = lane & 7, koff = (lane >> 3) & 1;
            ldsm_x2(a_base + row * A_PITCH + (s * 16 + koff * 8) * 2, b[0][0], b[0][1]);
          } else {
#pragma unroll
            for (int q = 0; q < NT8 / 2; ++q) {
              const int row = q * 16 + (lane & 7) + ((lane >> 4) << 3);
              const int koff = (lane >> 3) & 1;
              ldsm_x4(a_base + row * A_PITCH + (s * 16 + koff * 8) * 2, b[2 * q][0], b[2 * q][1], b[2 * q + 1][0],
                      b[2 * q + 1][1]);
            }
          }
          const int kglob = (kb0 + kbl) * TILE_K + s * 16;
          const int grp = kglob / p.group - g0;
#pragma unroll
          for (int pn = 0; pn < 4; ++pn) {
            const int rlo = pn * 16 + g, rhi = rlo + 8;
            uint32_t a[4];
            if constexpr (WF == W_INT4 || WF == W_UINT4) {
              const uint16_t *sc = reinterpret_cast<const uint16_t *>(sS) + grp * TILE_N;
              const uint32_t slo = bcast16(sc[rlo]), shi = bcast16(sc[rhi]);
              uint32_t zlo, zhi;
              if constexpr (WF == W_UINT4) {
                const uint8_t *zz = sS + SM::S + grp * TILE_N;
                zlo = bcast16(0x4300u + zz[rlo]);
                zhi = bcast16(0x4300u + zz[rhi]);
              } else {
                zlo = zhi = 0x43084308u;  // 128 + 8
              }
              const uint32_t w = (s == 0) ? wv[pn][0].x : (s == 1) ? wv[pn][0].y : (s == 2) ? wv[pn][0].z : wv[pn][0].w;
              dequant_int(w, zlo, zhi, slo, shi, a);
            } else if constexpr (T::fp4) {
              const uint32_t slo = bcast16(sSB[grp * TILE_N + rlo]), shi = bcast16(sSB[grp * TILE_N + rhi]);
              const uint32_t w = (s == 0) ? wv[pn][0].x : (s == 1) ? wv[pn][0].y : (s == 2) ? wv[pn][0].z : wv[pn][0].w;
              dequant_fp4(w, slo, shi, a);
            } else {
              const uint4 v = wv[pn][s >> 1];
              const uint32_t wa = (s & 1) ? v.z : v.x;
              const uint32_t wb2 = (s & 1) ? v.w : v.y;
              dequant_fp8(wa, wb2, a);
            }
#pragma unroll
            for (int j = 0; j < NT8; ++j) mma_bf16(acc[pn][j], a, b[j][0], b[j][1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stg]);
    }
    // all consumers done with the ring before it is reused for the reduction
    asm volatile("bar.sync 1, %0;" ::"n"(CONSUMERS * 32));
    float *red = reinterpret_cast<float *>(smem);
    const int t4 = lane & 3;
#pragma unroll
    for (int pn = 0; pn < 4; ++pn)
#pragma unroll
      for (int j = 0; j < NT8; ++j) {
        const int r0 = pn * 16 + g, c0 = j * 8 + 2 * t4;
        float *rw = red + (size_t)warp * TILE_N * (MT + 1);
        rw[r0 * (MT + 1) + c0] = acc[pn][j][0];
        rw[r0 * (MT + 1) + c0 + 1] = acc[pn][j][1];
        rw[(r0 + 8) * (MT + 1) + c0] = acc[pn][j][2];
        rw[(r0 + 8) * (MT + 1) + c0 + 1] = acc[pn][j][3];
      }
  }
  __syncthreads();

  // ---- reduction over warps, split-K fixup, epilogue ----
  float *red = reinterpret_cast<float *>(smem);
  const int n_l = tid & 63;
  const int n = nt * TILE_N + n_l;
  const int tile = slot * p.NT + nt;
  constexpr int MPT = (MT + 1) / 2;  // tokens per thread (two thread groups of 64)
  float v[MPT];
  if (tid < 128) {
#pragma unroll
    for (int q = 0; q < MPT; ++q) {
      const int m = (tid >> 6) + 2 * q;
      float s = 0.f;
      if (m < MT) {
#pragma unroll
        for (int w = 0; w < CONSUMERS; ++w) s += red[(size_t)w * TILE_N * (MT + 1) + n_l * (MT + 1) + m];
      }
      v[q] = s;
    }
  }
  bool write = true;
  if (p.splits > 1) {
    float *part = p.partial + ((size_t)tile * p.splits + split) * MT * TILE_N;
    if (tid < 128) {
#pragma unroll
      for (int q = 0; q < MPT; ++q) {
        const int m = (tid >> 6) + 2 * q;
        if (m < MT) __stcg(&part[m * TILE_N + n_l], v[q]);
      }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const int ticket = atomicAdd(&p.counters[tile], 1);
      s_info[2] = (ticket == p.splits - 1);
    }
    __syncthreads();
    write = s_info[2] != 0;
    if (write) {
      __threadfence();
      if (tid < 128) {
#pragma unroll
        for (int q = 0; q < MPT; ++q) {
          const int m = (tid >> 6) + 2 * q;
          float s = 0.f;
          if (m < MT) {
            const float *pp = p.partial + (size_t)tile * p.splits * MT * TILE_N + m * TILE_N + n_l;
            for (int sp = 0; sp < p.splits; ++sp) s += __ldcg(pp + (size_t)sp * MT * TILE_N);
          }
          v[q] = s;
        }
      }
      if (tid == 0) p.counters[tile] = 0;  // ready for the next call
    }
  }
  if (write && tid < 128 && n < p.N) {
    float cs = 1.f;
    if constexpr (WF == W_FP8) cs = reinterpret_cast<const float *>(eb + p.c_off)[(size_t)nt * TILE_N + n_l];
    float gs = 1.f;
    if constexpr (WF == W_NVFP4) gs = reinterpret_cast<const float *>(eb + p.g_off)[0];
    if (p.a_global) gs = __fmul_rn(gs, *p.a_global);
#pragma unroll
    for (int q = 0; q < MPT; ++q) {
      const int m = (tid >> 6) + 2 * q;
      if (m < MT && m < nvalid) {
        float r = v[q];
        if (p.row_scale) r *= p.row_scale[s_srow[m]];
        r *= cs;
        r *= gs;
        p.out[(size_t)s_orow[m] * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(r));
      }
    }
  }
}

// ---- host-side launch ---------------------------------------------------------
// Chooses the token tile and the split-K factor so that the grid covers the
// 148 SMs about twice.
StreamLaunch plan_stream(int rows_bound, int mtiles_bound_moe, int NT, int KB, bool moe) {
  StreamLaunch s{};
  s.mt = rows_bound <= 8 ? 8 : rows_bound <= 16 ? 16 : 32;
  s.mtiles = moe ? mtiles_bound_moe : (rows_bound + s.mt - 1) / s.mt;
  if (s.mtiles < 1) s.mtiles = 1;
  const long tiles = (long)NT * s.mtiles;
  const long target = 2 * 148;
  int splits = (int)((target + tiles - 1) / tiles);
  const int max_splits = (KB + S_KB - 1) / S_KB;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  // whole stages per split
  int kbps = (KB + splits - 1) / splits;
  kbps = (kbps + S_KB - 1) / S_KB * S_KB;
  splits = (KB + kbps - 1) / kbps;
  s.splits = splits;
  s.kb_per_split = kbps;
  return s;
}

size_t stream_workspace_bytes(const StreamLaunch &s, int NT) {
  if (s.splits <= 1) return 256;
  const size_t tiles = (size_t)NT * s.mtiles;
  return align_up(tiles * sizeof(int), 256) + tiles * s.splits * s.mt * TILE_N * sizeof(float);
}

template <int WF, int MT>
static hq_status launch_one(const StreamParams &p, const StreamLaunch &s, cudaStream_t st) {
  using SM = Smem<WF, MT>;
  auto kern = stream_gemm_kernel<WF, MT>;
  static unsigned configured = 0;  // one bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
  if (dev >= 32 || !(configured & (1u << dev))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SM::BYTES) != cudaSuccess)
      return HQ_ERR_CUDA;
    if (dev < 32) configured |= 1u << dev;
  }
  dim3 grid(p.NT * s.splits, s.mtiles);
  kern<<<grid, THREADS, SM::BYTES, st>>>(p);
  return check_launch();
}

template <int WF>
static hq_status launch_wf(const StreamParams &p, const StreamLaunch &s, cudaStream_t st) {
  switch (s.mt) {
    case 8: return launch_one<WF, 8>(p, s, st);
    case 16: return launch_one<WF, 16>(p, s, st);
    default: return launch_one<WF, 32>(p, s, st);
  }
}

hq_status launch_stream_gemm(const Layout &L, const void *packed, const void *a_bf16, const float *row_scale,
                             const float *a_global, int M, int moe, int E, const int32_t *offsets,
                             const int32_t *perm, int a_indexed, int a_div, void *out, const StreamLaunch &s,
                             void *workspace, cudaStream_t st) {
  StreamParams p{};
  p.packed = (const uint8_t *)packed;
  p.stride = L.stride;
  p.w_off = L.w_off; p.s_off = L.s_off; p.z_off = L.z_off; p.c_off = L.c_off; p.g_off = L.g_off;
  p.N = L.N; p.K = L.K; p.NT = L.NT; p.KB = L.KB; p.G = L.G; p.group = L.group;
  p.a = (const uint16_t *)a_bf16;
  p.row_scale = row_scale;
  p.a_global = a_global;
  p.M = M;
  p.moe = moe;
  p.E = E;
  p.offsets = offsets;
  p.perm = perm;
  p.a_indexed = a_indexed;
  p.a_div = a_div;
  p.out = (uint16_t *)out;
  p.splits = s.splits;
  p.kb_per_split = s.kb_per_split;
  if (s.splits > 1) {
    const size_t tiles = (size_t)L.NT * s.mtiles;
    p.counters = (int *)workspace;
    p.partial = (float *)((uint8_t *)workspace + align_up(tiles * sizeof(int), 256));
  }
  switch (L.fmt) {
    case W_INT4: return launch_wf<W_INT4>(p, s, st);
    case W_UINT4: return launch_wf<W_UINT4>(p, s, st);
    case W_MXFP4: return launch_wf<W_MXFP4>(p, s, st);
    case W_NVFP4: return launch_wf<W_NVFP4>(p, s, st);
    case W_FP8: return launch_wf<W_FP8>(p, s, st);
    default: return HQ_ERR_UNSUPPORTED;
  }
}

}  // namespace hq
