// Internal definitions shared by the sm_100a kernels of libhq.
//
// Packed weight layout (the "repack into the kernel's layout" step of
// "Announcing Humming", section "Tuning and JIT compilation per workload").
// Per expert, 256-byte aligned regions:
//
//   weights  [NT][KB][CH][128 rows][16 B]   CH = 2 chunks of 32 k (4-bit)
//                                           or 4 chunks of 16 k (8-bit)
//   scales   [NT][G][128]  element = bf16 | E8M0 | UE4M3 (one group =
//                          w_group k's; per-channel scales use G = 1)
//   zeros    [NT][G][128]  uint8 (UINT4 only)
//   chscale  [NT][128]     fp32 (FP8 per-channel scales)
//   global   fp32          (NVFP4 second-level scale)
//
// with NT = ceil(N / 128) row tiles and KB = K / 64 k-blocks.  One (row
// tile, k-block) unit is contiguous (4 KiB for 4-bit, 8 KiB for 8-bit), so a
// CTA streams it with one bulk copy; inside it, thread r of the dequant
// warps reads the 16-byte chunks of row r, consecutive threads consecutive
// 16 bytes (conflict-free).  Within a 32-bit word the values are interleaved
// so that one mask yields an adjacent k pair in the two bf16 halves:
//   4-bit: nibble p holds k offset 2*(p%4) + p/4, so (w >> 4i) & 0x000F000F
//          is the pair (k 2i, k 2i+1);
//   8-bit: bytes hold k offsets [0 2 1 3], so (w >> 8i) & 0x00FF00FF is the
//          pair (k 2i, k 2i+1).
// INT4 codes are stored biased (u = q + 8) so every integer format decodes
// as (u - z); signed INT4 uses z = 8.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hq.h"

namespace hq {

// Internal weight formats.
// W_MXINT4: INT4 codes with an E8M0 scale per 32 along K (the MX layout with
// integer elements).  Low-bit WnA16 widths: W_INT2 / W_INT3 (signed, stored
// biased like INT4), W_UINT2 / W_UINT3 (with zero points), W_E2M3 / W_E3M2
// (MXFP6, E8M0 per 32).  W_E0M3 (float4e0m3, the zero-exponent view of
// symmetric INT4) is converted by the repack into the INT4 layout; the GEMM
// kernels see INT4.
enum WFmt : int {
  W_INT4 = 0, W_UINT4 = 1, W_MXFP4 = 2, W_NVFP4 = 3, W_FP8 = 4, W_MXINT4 = 5,
  W_INT2 = 6, W_UINT2 = 7, W_INT3 = 8, W_UINT3 = 9, W_E2M3 = 10, W_E3M2 = 11, W_E0M3 = 12,
  W_FP8B = 13,  // E4M3 with one fp32 scale per 128 x 128 block (rows x k)
  W_INT1 = 14, W_UINT1 = 15,
  W_NFMT = 16
};

// Bits per stored weight code of a format.
__host__ __device__ constexpr int fmt_bits(int fmt) {
  return (fmt == W_FP8 || fmt == W_FP8B) ? 8 : (fmt == W_INT2 || fmt == W_UINT2) ? 2 : (fmt == W_INT3 || fmt == W_UINT3) ? 3
         : (fmt == W_E2M3 || fmt == W_E3M2) ? 6 : (fmt == W_INT1 || fmt == W_UINT1) ? 1 : 4;
}
__host__ __device__ constexpr bool fmt_lowbit(int fmt) {
  return (fmt >= W_INT2 && fmt <= W_E3M2) || fmt == W_INT1 || fmt == W_UINT1;
}
__host__ __device__ constexpr bool fmt_zero(int fmt) {
  return fmt == W_UINT4 || fmt == W_UINT2 || fmt == W_UINT3 || fmt == W_UINT1;
}
__host__ __device__ constexpr bool fmt_bf16_scales(int fmt) {
  return fmt == W_INT4 || fmt == W_UINT4 || fmt == W_INT2 || fmt == W_UINT2 || fmt == W_INT3 || fmt == W_UINT3 ||
         fmt == W_E0M3 || fmt == W_INT1 || fmt == W_UINT1;
}
// Unit planes of the low-bit layouts (byte offsets inside a 128-row x 64-k
// unit): a 4-bit plane (the INT4 unit's order, 4 KiB; 6-bit codes' low
// nibbles), a 2-bit plane ([128 rows][16 B]: word j of a row holds k
// 16j..16j+15, even k in bits 0..15 and odd k in bits 16..31, two bits
// each; the low two bits of 2- and 3-bit codes, the high two of 6-bit
// ones) and a 1-bit plane ([128 rows][8 B]: word j holds k 32j..32j+31,
// even k in bits 0..15, odd in 16..31; the high bit of 3-bit codes, or the
// 1-bit codes themselves).
__host__ __device__ constexpr int plane2_off(int fmt) { return (fmt == W_E2M3 || fmt == W_E3M2) ? 4096 : 0; }
__host__ __device__ constexpr int plane1_off(int fmt) { return (fmt == W_INT3 || fmt == W_UINT3) ? 2048 : 0; }
// Internal activation formats (A_FP8G: E4M3 with an fp32 scale per token and
// 128 k).
enum AFmt : int { A_BF16 = 0, A_FP8 = 1, A_MXFP8 = 2, A_NVFP4 = 3, A_FP8G = 4 };

constexpr int TILE_N = 128;  // rows of W per tile (the MMA M dimension)
constexpr int TILE_K = 64;   // k per k-block

// Block-scaled layouts: weights that the tensor core consumes as they are
// (no dequantisation), with the block scales next to them.
enum { BS_NONE = 0, BS_MX = 1, BS_NV = 2, BS_F8 = 3, BS_F8B = 4 };

struct Layout {
  int fmt;
  int bs;                      // BS_*: block-scaled MMA layout, or the dequantisation layout
  int gated;                   // gate-up weights for the fused SiLU-and-mul epilogue (see std_row)
  int N, K, NT, KB, G, group;  // group = k per scale group (K for per-channel)
  int wbits;                   // 4 or 8
  int sbytes;                  // bytes per scale element (per-group scales)
  size_t w_bytes, s_bytes, z_bytes, c_bytes, g_bytes;  // per expert
  size_t w_off, s_off, z_off, c_off, g_off, stride;     // offsets inside an expert region
  __host__ __device__ size_t unit_bytes() const { return (size_t)TILE_N * TILE_K * wbits / 8; }
  // Gate-up weights (N = 2I rows: gate rows 0..I-1, then up rows) are packed
  // with the gate and the up row of output column j side by side: rows 2i
  // and 2i + 1 of 128-row tile t hold gate and up rows of column 64 t + i,
  // so one tile's epilogue has both values of 64 columns.  std_row maps a
  // packed row to its standard-format row, packed_row the other way.
  __host__ __device__ int std_row(int p) const {
    if (!gated) return p;
    const int i = p % TILE_N;
    return (p / TILE_N) * (TILE_N / 2) + (i >> 1) + ((i & 1) ? N / 2 : 0);
  }
  __host__ __device__ int packed_row(int r) const {
    if (!gated) return r;
    const int h = r >= N / 2 ? 1 : 0, j = h ? r - N / 2 : r;
    return (j / (TILE_N / 2)) * TILE_N + (j % (TILE_N / 2)) * 2 + h;
  }
  __host__ __device__ int chunks() const { return wbits == 4 ? 2 : 4; }
  // code bytes per weight row of the block-scaled / FP8 layouts
  __host__ __device__ size_t bs_row_bytes() const { return (bs == BS_F8 || bs == BS_F8B) ? (size_t)K : (size_t)K / 2; }
  // ... stored in chunks of this many bytes per row: one MMA stage (MX: 128
  // codes = 64 bytes; NV: 256 codes, F8: 128 codes = 128 bytes)
  __host__ __device__ int bs_chunk_bytes() const { return bs == BS_MX ? 64 : 128; }
  // byte offset (from w_off) of row r's chunk c: [NT][row_bytes / chunk][128 rows][chunk]
  __host__ __device__ size_t bs_chunk_off(int r, int c) const {
    const size_t nc = bs_row_bytes() / bs_chunk_bytes();
    return (((size_t)(r / TILE_N) * nc + c) * TILE_N + (r % TILE_N)) * bs_chunk_bytes();
  }
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Returns false if the description is not one of the supported ones.
inline bool weight_format(const hq_quant_desc *d, int *fmt) {
  if (!d) return false;
  switch (d->w_dtype) {
    case HQ_INT4:
      if (d->w_has_zero || d->w_has_global) return false;
      if (d->w_scale_dtype == HQ_E8M0) {
        if (d->w_group != 32) return false;
        *fmt = W_MXINT4;
        return true;
      }
      if (d->w_scale_dtype != HQ_BF16) return false;
      if (!(d->w_group == 0 || d->w_group == 32 || d->w_group == 64 || d->w_group == 128)) return false;
      *fmt = W_INT4;
      return true;
    case HQ_UINT4:
      if (d->w_scale_dtype != HQ_BF16 || !d->w_has_zero || d->w_has_global) return false;
      if (!(d->w_group == 32 || d->w_group == 64 || d->w_group == 128)) return false;
      *fmt = W_UINT4;
      return true;
    case HQ_E2M1:
      if (d->w_has_zero) return false;
      if (d->w_scale_dtype == HQ_E8M0 && d->w_group == 32 && !d->w_has_global) { *fmt = W_MXFP4; return true; }
      if (d->w_scale_dtype == HQ_UE4M3 && d->w_group == 16 && d->w_has_global) { *fmt = W_NVFP4; return true; }
      return false;
    case HQ_E4M3:
      if (d->w_scale_dtype != HQ_FP32 || d->w_has_zero || d->w_has_global) return false;
      if (d->w_group == 128) { *fmt = W_FP8B; return true; }  // 128 x 128 blocks
      if (d->w_group != 0) return false;
      *fmt = W_FP8;
      return true;
    case HQ_INT1:
    case HQ_INT2:
    case HQ_INT3:
    case HQ_E0M3:
      if (d->w_scale_dtype != HQ_BF16 || d->w_has_zero || d->w_has_global) return false;
      if (!(d->w_group == 0 || d->w_group == 32 || d->w_group == 64 || d->w_group == 128)) return false;
      *fmt = d->w_dtype == HQ_INT1 ? W_INT1 : d->w_dtype == HQ_INT2 ? W_INT2 : d->w_dtype == HQ_INT3 ? W_INT3 : W_E0M3;
      return true;
    case HQ_UINT1:
    case HQ_UINT2:
    case HQ_UINT3:
      if (d->w_scale_dtype != HQ_BF16 || !d->w_has_zero || d->w_has_global) return false;
      if (!(d->w_group == 32 || d->w_group == 64 || d->w_group == 128)) return false;
      *fmt = d->w_dtype == HQ_UINT1 ? W_UINT1 : d->w_dtype == HQ_UINT2 ? W_UINT2 : W_UINT3;
      return true;
    case HQ_E2M3:
    case HQ_E3M2:
      if (d->w_scale_dtype != HQ_E8M0 || d->w_group != 32 || d->w_has_zero || d->w_has_global) return false;
      *fmt = d->w_dtype == HQ_E2M3 ? W_E2M3 : W_E3M2;
      return true;
    default:
      return false;
  }
}

// K must hold whole k-blocks and whole scale groups.
inline bool valid_k(const hq_quant_desc *d, int K) {
  if (K < 64 || (K % 64) != 0) return false;
  return d->w_group == 0 || (K % d->w_group) == 0;
}

// The activation format of a description; a_group must be 0 (the format's
// own scale granularity) or that granularity spelled out.
inline bool act_format(const hq_quant_desc *d, int *afmt) {
  switch (d->a_dtype) {
    case HQ_BF16: *afmt = A_BF16; return d->a_group == 0;
    case HQ_E4M3:
      *afmt = d->a_group == 128 ? A_FP8G : A_FP8;
      return d->a_group == 0 || d->a_group == 128;
    case HQ_MXFP8: *afmt = A_MXFP8; return d->a_group == 0 || d->a_group == 32;
    case HQ_NVFP4: *afmt = A_NVFP4; return d->a_group == 0 || d->a_group == 16;
    default: return false;
  }
}

// Packed layouts.
//  * Dequantisation layout (bs == BS_NONE): see the unit description above.
//  * Block-scaled layouts, chosen when the activation format makes the pair
//    one the tensor core multiplies with block scales itself:
//      BS_MX  MXFP4 weights x MXFP8 activations (kind::mxf8f6f4, K % 128 == 0)
//      BS_NV  NVFP4 weights x NVFP4 activations (kind::mxf4nvf4, K % 256 == 0)
//    codes: [NT][stages][128 rows][chunk] bytes, two E2M1 codes per byte
//    (even k in the low nibble), rows past N zero, chunk = one stage of a row
//    (MX: 64 bytes, NV: 128 bytes), so that a stage of a tile is one
//    contiguous 8 / 16 KB piece of HBM; scales: per 128-row tile, chunks of
//    4 scale columns x 128 rows in the order the tensor-memory copy expects
//    (row i, scale column j of the chunk at byte (i%32)*16 + (i/32)*4 + j),
//    [NT][K / (4 * scale group)][512 B]; NVFP4 global scale as fp32.
//  * BS_F8: FP8 weights x FP8 activations with K % 128 == 0 (kind::f8f6f4,
//    both operands straight from TMA): codes [NT][K/128][128 rows][128 B]
//    E4M3 bytes, rows past N zero; per-row fp32 scales [NT*128] (zero past N).
inline Layout make_layout(int fmt, int group, int N, int K, int bs = BS_NONE) {
  Layout L{};
  L.fmt = fmt;
  L.bs = bs;
  L.N = N;
  L.K = K;
  L.NT = (N + TILE_N - 1) / TILE_N;
  L.KB = K / TILE_K;
  L.group = (group == 0) ? K : group;
  L.G = K / L.group;
  L.wbits = fmt_bits(fmt);
  L.sbytes = fmt_bf16_scales(fmt) ? 2 : 1;
  L.w_bytes = (size_t)L.NT * L.KB * L.unit_bytes();
  L.s_bytes = (fmt == W_FP8) ? 0 : (size_t)L.NT * L.G * TILE_N * L.sbytes;
  L.z_bytes = fmt_zero(fmt) ? (size_t)L.NT * L.G * TILE_N : 0;
  if (fmt == W_FP8B) L.s_bytes = 0;
  L.c_bytes = (fmt == W_FP8) ? (size_t)L.NT * TILE_N * 4 : 0;
  L.g_bytes = (fmt == W_NVFP4) ? 16 : 0;
  if (bs != BS_NONE) {
    L.w_bytes = (size_t)L.NT * TILE_N * L.bs_row_bytes();
    L.s_bytes = (bs == BS_F8 || bs == BS_F8B) ? 0 : (size_t)L.NT * (K / (4 * L.group)) * 512;
    L.z_bytes = 0;
    L.c_bytes = bs == BS_F8 ? (size_t)L.NT * TILE_N * 4 : bs == BS_F8B ? (size_t)L.NT * (K / 128) * 4 : 0;
  }
  size_t off = 0;
  L.w_off = off; off = align_up(off + L.w_bytes, 256);
  L.s_off = off; off = align_up(off + L.s_bytes, 256);
  L.z_off = off; off = align_up(off + L.z_bytes, 256);
  L.c_off = off; off = align_up(off + L.c_bytes, 256);
  L.g_off = off; off = align_up(off + L.g_bytes, 256);
  L.stride = off;
  return L;
}

// The packed layout of a description: block-scaled when the weight and
// activation formats pair up for a block-scaled MMA and K fits its stage.
inline Layout layout_for(const hq_quant_desc *d, int fmt, int N, int K) {
  int afmt = -1;
  int bs = BS_NONE;
  if (act_format(d, &afmt)) {
    if (fmt == W_MXFP4 && afmt == A_MXFP8 && (K % 128) == 0) bs = BS_MX;
    if (fmt == W_NVFP4 && afmt == A_NVFP4 && (K % 256) == 0) bs = BS_NV;
    if (fmt == W_FP8 && afmt == A_FP8 && (K % 128) == 0) bs = BS_F8;
    if (fmt == W_FP8B && afmt == A_FP8G && (K % 128) == 0) bs = BS_F8B;
  }
  return make_layout(fmt, d->w_group, N, K, bs);
}

// Formats that exist only as a pair: block-scaled FP8 weights with per-128
// FP8 activations (the block-scaled W8A8 of DeepGEMM-style MoE), on the
// TMA-fed kernel.
inline bool pair_supported(const Layout &L, int afmt) {
  if (L.fmt == W_FP8B || afmt == A_FP8G) return L.bs == BS_F8B;
  return true;
}

// Device-side error word (one per device, module scope).  The library is
// built as one translation unit (libhq.cu), so the definition lives here.
__device__ int g_hq_error = 0;

// Polling bound for every device-side wait: about one second.
constexpr unsigned long long WAIT_LIMIT_NS = 1000000000ull;

#ifdef __CUDACC__
__device__ __forceinline__ void set_device_error(int code) { atomicCAS(&g_hq_error, 0, code); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps until the phase
// completes or about `hint_ns` have passed, instead of spinning and taking
// issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait: returns false (and records HQ_ERR_TIMEOUT) after about a
// second without the phase completing.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          unsigned long long limit_ns = WAIT_LIMIT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      set_device_error(HQ_ERR_TIMEOUT);
      return false;
    }
  }
}

// 1-D bulk copy global -> shared, completing on an mbarrier (16-byte
// aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Same, with an L2 evict-first hint for data read exactly once (weights).
__device__ __forceinline__ void bulk_g2s_stream(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                                uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
      "%4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
#endif

// Launch plan of the tensor-core GEMM (hq_gemm_tc.cu).
struct TcLaunch {
  int kind;    // 0: multi-CTA-per-SM kernel (>= 64 tokens per tile); 1: decode kernel (16 or 32);
               // 2: block-scaled kernel (16..128)
  int bnt;     // token tile = MMA N (16, 32, 64, 128, 256)
  int ntw;     // 128-row weight tiles
  int mtiles;  // token tiles (dense) or an upper bound on (expert, tile) pairs (MoE)
  int nctas;   // persistent CTAs
};
TcLaunch plan_tc(int rows_per_tile, int mtiles_bound_moe, int N, int KB, bool moe, int bs = BS_NONE);
size_t tc_workspace_bytes(const TcLaunch &t);
// Bytes at the head of the workspace that must be zero before the first
// call (tile tickets; every call leaves them zero again).
size_t tc_counter_bytes(const TcLaunch &t);

// Host-side helpers implemented in hq_api.cu.
hq_status check_launch();
bool device_is_sm100();

}  // namespace hq
