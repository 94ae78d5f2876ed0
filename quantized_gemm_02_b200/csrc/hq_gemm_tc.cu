// Tensor-core (tcgen05 / TMEM) quantised-weight GEMM, dense and MoE, for
// every token count.
//
// "Announcing Humming", section "Tuning and JIT compilation per workload":
// a TMA + UMMA pipeline with dequantisation and scaling fused into the kernel
// ("Shared CUDA components across formats and architectures"), work split
// along K for small batches.  The sm_100a design:
//
//   * swap-AB: 128 weight rows are the MMA's M side and sit in TENSOR MEMORY
//     as operand A; a tile of 16..256 tokens is the N side, operand B, in
//     shared memory.  Dequantised weights never touch shared memory, so the
//     shared-memory traffic per packed weight byte stays at ~2 bytes even
//     when the kernel streams weights at full HBM rate;
//   * warp roles (14 warps):
//       warps 0..3   epilogue: tcgen05.ld of the fp32 accumulator (warp w owns
//                    TMEM lanes 32w..32w+31), fp32 scales, bf16 out or fp32
//                    split-K partials with a deterministic last-split fixup;
//       warp 4       producer: TMA of the activation tile (bf16, 128-byte
//                    swizzle; for MoE indexed mode 4-row gathers of the
//                    caller's rows through the routing index), 1-D bulk
//                    copies of the packed weight unit, scales, zero points;
//       warp 5       MMA issuer: tcgen05.mma.cta_group::1.kind::f16 with A
//                    from TMEM and B from a shared-memory descriptor;
//       warps 6..13  dequant: thread = weight row, decodes 32 k of its row per
//                    k-block to bf16 pairs and stores them with
//                    tcgen05.st.32x32b into the A ring in TMEM;
//   * persistent CTAs (one or two per SM): whole tiles round-robin when
//     there are at least as many tiles as CTAs, else K-split units with a
//     deterministic fp32 fixup by the last split of each tile;
//   * shared-memory ring (NS stages of up to KPS 64-k blocks) for
//     activations and packed weights, TMEM ring (NA blocks of 32 columns,
//     16 for E4M3) for dequantised weights, fp32 accumulators (two where
//     TMEM allows) after the ring;
//   * every mbarrier wait is bounded (~1 s); on a timeout the CTA records
//     HQ_ERR_TIMEOUT, raises an abort flag, releases its TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "hq_internal.cuh"

namespace hq {

namespace tc {

constexpr int BM = TILE_N;        // 128 weight rows = MMA M
constexpr int THREADS = 14 * 32;
constexpr int WARP_PRODUCER = 4, WARP_MMA = 5, WARP_DQ0 = 6, NDQ = 8;

template <int WF>
struct Traits {
  static constexpr int wbits = fmt_bits(WF);
  static constexpr int unit = BM * TILE_K * wbits / 8;  // packed bytes per (tile, k-block)
  static constexpr int sbytes = fmt_bf16_scales(WF) ? 2 : 1;
  static constexpr int max_groups_kb = (WF == W_NVFP4) ? 4 : 2;  // scale groups per k-block (upper bound)
  static constexpr bool has_scales = (WF != W_FP8);
  static constexpr bool has_zero = fmt_zero(WF);
};

// F8: both operands E4M3 (kind::f8f6f4, weights copied into TMEM unchanged);
// otherwise weights are dequantised to bf16 (kind::f16).
// F8: both operands E4M3 (kind::f8f6f4, weights copied into TMEM unchanged);
// otherwise weights are dequantised to bf16 (kind::f16).
template <int WF, int BNT, bool F8>
struct Cfg {
  static constexpr int KPS = BNT <= 16 ? 4 : BNT <= 64 ? 2 : BNT <= 128 ? 3 : 1;  // 64-k blocks per stage
  static constexpr int A_COLS = F8 ? 16 : 32;                                  // TMEM columns per 64-k block
  static constexpr int ACT_KB = BNT * (F8 ? 64 : 128);                         // one block of activations
  static constexpr int ACT = KPS * ACT_KB;                                     // [KPS][BNT][64], swizzled
  static constexpr int WPK = KPS * Traits<WF>::unit;
  static constexpr int SC = KPS * Traits<WF>::max_groups_kb * BM * Traits<WF>::sbytes;
  static constexpr int ZP = Traits<WF>::has_zero ? KPS * Traits<WF>::max_groups_kb * BM : 0;
  static constexpr int STAGE = (ACT + WPK + SC + ZP + 1023) / 1024 * 1024;
  // two CTAs per SM up to 64 tokens (TMEM 2 x 256 columns), one beyond
  static constexpr int CTAS_PER_SM = BNT <= 64 ? 2 : 1;
  static constexpr int NS_BY_SMEM = ((CTAS_PER_SM == 2 ? 100 : 196) * 1024) / STAGE;
  static constexpr int NS = NS_BY_SMEM > 8 ? 8 : NS_BY_SMEM;                  // shared-memory ring depth
  static constexpr int CTRL = 8192;                                            // barriers + tile tables
  static constexpr int BYTES = NS * STAGE + CTRL + 1024;                      // + alignment slack
  // TMEM: the CTA's share (256 columns with two CTAs per SM, else 512) holds
  // ND accumulators of BNT columns and a ring of NA dequantised 64-k blocks.
  // The ring must cover the MMA completion latency (~1 us), so it takes all
  // the columns the accumulators leave.
  static constexpr int TMEM_COLS = CTAS_PER_SM == 2 ? 256 : 512;
  static constexpr int ND = (4 * A_COLS + 2 * BNT) <= TMEM_COLS ? 2 : 1;      // accumulator buffers
  static constexpr int NA_FIT = (TMEM_COLS - ND * BNT) / A_COLS;
  static constexpr int NA = NA_FIT > 12 ? 12 : NA_FIT;                         // TMEM A ring depth
  static constexpr int D_COL = NA * A_COLS;                                    // accumulators start
  static_assert(NS >= 2, "stage too large");
  static_assert(NA >= 2 && D_COL + ND * BNT <= TMEM_COLS, "TMEM budget");
};

struct Params {
  const uint8_t *packed;
  size_t stride;
  size_t w_off, s_off, z_off, c_off, g_off;
  int N, K, NT, KB, G, group;
  int gshift;              // k >> gshift = scale group (31 for one group per row)
  const float *row_scale;  // per caller row (FP8 per-token) or null
  const float *a_global;   // NVFP4 activation global scale or null
  int gated;               // fused SiLU-and-mul: out[row, n / 2] = silu(gate) * up (packed rows 2j, 2j + 1)
  int M;                   // dense rows
  int moe, E;
  const int32_t *offsets, *perm;
  int a_div;
  int gather;              // MoE indexed mode: activation rows gathered by index
  uint16_t *out;
  int ntw;                 // 128-row weight tiles
  int mtiles;              // token tiles (dense: exact; MoE: upper bound)
  int nctas;               // persistent CTAs (grid size)
  int weights_once;        // every weight tile is read by one token tile only (stream it past L2)
  int group_slots;         // dense: token tiles per raster group (<= 1: weight tile fastest)
  const uint8_t *a_sf;     // block-scaled kernel: activation block scales, a_sf_ld bytes per row
  int a_sf_ld;
  int a_rows;              // block-scaled kernel: rows of the activation matrix
  float *partial;          // [tiles * S][BNT][128] fp32 split-K partial tiles
  int *counters;           // [ntw * mtiles] per-tile arrival tickets
};

// ---- PTX wrappers ----------------------------------------------------------------
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;            // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset: 8-row groups 1024 B apart
  d |= (uint64_t)1 << 46;            // descriptor version
  d |= (uint64_t)2 << 61;            // 128-byte swizzle
  return d;
}

// K-major, 64-byte swizzle (rows of 64 e4m3 codes, 8-row groups 512 B apart)
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(512 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)4 << 61;  // 64-byte swizzle
  return d;
}

template <int BNT>
__device__ __forceinline__ constexpr uint32_t idesc_e4m3() {
  return (1u << 4)                       // D = f32; A = B = E4M3 (format 0)
         | ((uint32_t)(BNT >> 3) << 17)  // N
         | ((uint32_t)(BM >> 4) << 24);  // M
}

template <int BNT>
__device__ __forceinline__ constexpr uint32_t idesc_bf16() {
  return (1u << 4)                       // D = f32
         | (1u << 7) | (1u << 10)        // A = B = bf16
         | ((uint32_t)(BNT >> 3) << 17)  // N
         | ((uint32_t)(BM >> 4) << 24);  // M
}

__device__ __forceinline__ void mma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_ts_f8(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                          uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Four rows (given by index) of one box column of a 2-D tensor map with
// one-row boxes, landing as consecutive box rows in shared memory.
__device__ __forceinline__ void tma_gather4(void *dst, const CUtensorMap *map, int x, int r0, int r1, int r2, int r3,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// ---- output ---------------------------------------------------------------------
// silu(g) * u in fp32 (CUDA expf, IEEE division), as hq_silu_and_mul computes it.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fmul_rn(__fdiv_rn(g, __fadd_rn(1.f, expf(-g))), u);
}

// One scaled output value of weight row n for output row `orow`.  Plain: bf16
// at column n.  Gated (gate-up weights packed gate/up side by side): lanes of
// rows 2j and 2j + 1 exchange their values and the even lane writes
// silu(gate) * up at column n / 2 of an N / 2-wide row.  All 32 lanes of the
// warp call it together (consecutive lanes = consecutive weight rows).
// The epilogues pick the form once per block of stores (GatedTag<p.gated>),
// so that the plain stores of a block issue back to back.
template <bool G>
struct GatedTag {
  static constexpr bool value = G;
};
template <bool G>
__device__ __forceinline__ void put_out(const Params &p, int orow, int n, float z, bool ok) {
  if constexpr (!G) {
    if (ok) p.out[(size_t)orow * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(z));
  } else {
    const float u = __shfl_xor_sync(0xffffffffu, z, 1);
    if (ok && !(n & 1))
      p.out[(size_t)orow * (p.N >> 1) + (n >> 1)] = __bfloat16_as_ushort(__float2bfloat16_rn(silu_mul(z, u)));
  }
}

// ---- bf16 pair arithmetic and decoders ---------------------------------------
__device__ __forceinline__ uint32_t bsub2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162 *>(&a), *reinterpret_cast<__nv_bfloat162 *>(&b));
  return *reinterpret_cast<uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162 *>(&a), *reinterpret_cast<__nv_bfloat162 *>(&b));
  return *reinterpret_cast<uint32_t *>(&r);
}
__device__ __forceinline__ uint32_t bcast16(uint32_t h) { return (h & 0xFFFFu) * 0x10001u; }
// bf16 bits of an E4M3 / UE4M3 code's value (exact: <= 4 significant bits)
__device__ __forceinline__ uint32_t e4m3_code_to_bf16(uint32_t c) {
  const float mag = __uint_as_float((c & 0x7Fu) << 20) * 1.329227995784916e36f;  // 2^120
  return (__float_as_uint(mag) >> 16) | ((c & 0x80u) << 8);
}
// bf16 bits of 2^(c - 127) for an E8M0 code c in [0, 254]
__device__ __forceinline__ uint32_t e8m0_code_to_bf16(uint32_t c) { return c ? (c << 7) : 0x0040u; }
// E2M1 pair (codes at bits 0..3 and 16..19) -> bf16 pair carrying value * 2^-126
__device__ __forceinline__ uint32_t e2m1_pair(uint32_t x) {
  return ((x << 6) & 0x01C001C0u) | ((x << 12) & 0x80008000u);
}
// E4M3 pair (codes at bits 0..7 and 16..23) -> bf16 pair carrying value * 2^-120
__device__ __forceinline__ uint32_t e4m3_pair(uint32_t x) {
  return ((x & 0x007F007Fu) << 4) | ((x & 0x00800080u) << 8);
}

// Low-bit units (2-, 3- and 6-bit codes; planes as in hq_internal.cuh): the
// 32 k of half h (k 32h .. 32h + 31 of the 64-k block) of weight row r as 16
// bf16 pairs in k order (pair q = k 32h + 2q, 32h + 2q + 1).  Integer codes:
// ((u | 128) - (128 + z)) * s, the subtraction exact and the product the
// one rounding; MXFP6: the code's exponent and mantissa bits placed in the
// bf16 fields (the value times 2^-126 for E2M3, 2^-124 for E3M2, exact for
// subnormal codes too), scaled back, then by the E8M0 scale s2.
template <int WF>
__device__ __forceinline__ void decode_half_lowbit(const uint8_t *unit, uint32_t s2, uint32_t z2, int r, int h,
                                                   uint32_t *rg) {
  constexpr int b = fmt_bits(WF);
  uint32_t c[16];
  if constexpr (b == 1) {
    const uint32_t w1 = *reinterpret_cast<const uint32_t *>(unit + plane1_off(WF) + r * 8 + h * 4);
#pragma unroll
    for (int q = 0; q < 16; ++q) c[q] = (w1 >> q) & 0x00010001u;
  } else {
    const uint2 v2 = *reinterpret_cast<const uint2 *>(unit + plane2_off(WF) + r * 16 + h * 8);
    const uint32_t w2[2] = {v2.x, v2.y};
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int i = 0; i < 8; ++i) c[8 * a + i] = (w2[a] >> (2 * i)) & 0x00030003u;
  }
  if constexpr (b == 3) {
    const uint32_t w1 = *reinterpret_cast<const uint32_t *>(unit + plane1_off(WF) + r * 8 + h * 4);
#pragma unroll
    for (int q = 0; q < 16; ++q) c[q] |= ((w1 >> q) & 0x00010001u) << 2;
  }
  if constexpr (b == 6) {
    const uint4 v4 = *reinterpret_cast<const uint4 *>(unit + h * (BM * 16) + r * 16);
    const uint32_t w4[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int q = 0; q < 16; ++q) c[q] = (c[q] << 4) | ((w4[q >> 2] >> (4 * (q & 3))) & 0x000F000Fu);
  }
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    if constexpr (WF == W_E2M3) {
      const uint32_t x = ((c[q] & 0x001F001Fu) << 4) | ((c[q] & 0x00200020u) << 10);
      rg[q] = bmul2(bmul2(x, 0x7E807E80u), s2);  // x 2^126
    } else if constexpr (WF == W_E3M2) {
      const uint32_t x = ((c[q] & 0x001F001Fu) << 5) | ((c[q] & 0x00200020u) << 10);
      rg[q] = bmul2(bmul2(x, 0x7D807D80u), s2);  // x 2^124
    } else {
      rg[q] = bmul2(bsub2(c[q] | 0x43004300u, z2), s2);
    }
  }
}

// Scale and zero-point pairs of a low-bit row's group: bf16 scale (integer
// codes) or the E8M0 power of two (MXFP6); zero point 128 + z (unsigned
// codes) or 128 + 2^(b-1) (signed codes, stored biased).
template <int WF>
__device__ __forceinline__ void lowbit_scale_zero(const uint8_t *sc, const uint8_t *zp, int gt, int r, uint32_t &s2,
                                                  uint32_t &z2) {
  if constexpr (fmt_bf16_scales(WF)) s2 = bcast16(reinterpret_cast<const uint16_t *>(sc)[gt * BM + r]);
  else s2 = bcast16(e8m0_code_to_bf16(sc[gt * BM + r]));
  if constexpr (fmt_zero(WF)) z2 = bcast16(0x4300u + zp[gt * BM + r]);
  else z2 = bcast16(0x4300u + (1u << (fmt_bits(WF) - 1)));
}

// ---- the kernel ----------------------------------------------------------------
// Persistent CTAs.  Work units are (tile, k-range) pairs; tiles are ordered
// token-tile-major with the weight tile fastest.
//   * at least as many tiles as CTAs: unit u of CTA c is the whole tile
//     c + u * nctas (round-robin, so the CTAs running together share their
//     activation tile in L2 and no tile is shared between CTAs);
//   * fewer tiles than CTAs (decode sizes): every tile is split along K into
//     S contiguous ranges, one unit per CTA; each split stores an fp32
//     partial and the last split to arrive (atomic ticket) sums the S
//     partials in split order with all its threads.
// The TMEM accumulator is double-buffered where TMEM allows, so one unit's
// epilogue overlaps the next unit's main loop.

struct TileInfo {
  int wt, expert, base, nvalid;
};

struct Sched {
  int tiles;  // tiles in this call (MoE: from the routing)
  int S;      // K splits per tile (1 in round-robin mode)
  int kbps;   // k-blocks per split
  bool rr;    // round-robin whole tiles
};

__device__ __forceinline__ Sched make_sched(int tiles, int nctas, int KB) {
  Sched sc;
  sc.tiles = tiles;
  sc.rr = tiles >= nctas;
  if (sc.rr || tiles == 0) {
    sc.S = 1;
    sc.kbps = KB;
  } else {
    int S = nctas / tiles;
    const int max_s = KB / 2 > 0 ? KB / 2 : 1;  // at least two k-blocks per split
    if (S > max_s) S = max_s;
    sc.kbps = (KB + S - 1) / S;
    sc.S = (KB + sc.kbps - 1) / sc.kbps;
  }
  return sc;
}

// Unit u of CTA c: tile t, k-blocks [kb0, kb1) and split index; false once
// the CTA has no more work.
__device__ __forceinline__ bool unit_at(const Sched &sc, int c, int nctas, int KB, int u, int &t, int &kb0,
                                        int &kb1, int &split) {
  if (sc.rr) {
    t = c + u * nctas;
    if (t >= sc.tiles) return false;
    kb0 = 0;
    kb1 = KB;
    split = 0;
    return true;
  }
  if (u > 0 || c >= sc.tiles * sc.S) return false;
  t = c % sc.tiles;
  split = c / sc.tiles;
  kb0 = split * sc.kbps;
  kb1 = min(KB, kb0 + sc.kbps);
  return kb0 < kb1;
}

// A unit's k-blocks are walked in stages of KPS blocks, starting at a
// CTA-dependent stage and wrapping around, so that the CTAs running at the
// same time read different parts of the shared activation rows instead of
// all hitting the same L2 lines.  Every role walks the same order; the
// accumulation order is fixed by the CTA index, so results stay
// deterministic.
__device__ __forceinline__ int stage_rotation(int c, int nst) { return nst > 1 ? c % nst : 0; }
__device__ __forceinline__ int stage_of(int i, int rot, int nst) {
  const int s = i + rot;
  return s >= nst ? s - nst : s;
}

template <int WF, int BNT, bool F8>
__global__ void __launch_bounds__(THREADS, (BNT <= 64 ? 2 : 1)) tc_gemm_kernel(const __grid_constant__ CUtensorMap act_map,
                                                             const Params p) {
  using TR = Traits<WF>;
  using C = Cfg<WF, BNT, F8>;
  static_assert(!F8 || WF == W_FP8, "the E4M3 x E4M3 path takes FP8 weights");
  constexpr int NS = C::NS, ND = C::ND, NA = C::NA;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle, by offsetting from the
  // shared array itself so that the compiler keeps every access an ld.shared
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t *ctrl = smem + NS * C::STAGE;
  uint64_t *full = reinterpret_cast<uint64_t *>(ctrl);  // [NS] stage landed
  uint64_t *sfree = full + NS;                           // [NS] stage consumed (MMA + dequant)
  uint64_t *afull = sfree + NS;                          // [NA] TMEM A stage written
  uint64_t *aempty = afull + NA;                         // [NA] TMEM A stage consumed
  uint64_t *accf = aempty + NA;                          // [ND] accumulator complete
  uint64_t *acce = accf + ND;                            // [ND] accumulator drained
  long long *s_total = reinterpret_cast<long long *>(acce + ND);  // 8-byte slot after the barriers
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(s_total + 1);
  int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);
  int *s_last = s_abort + 1;
  int *s_tpre = s_last + 1;  // [E+1] MoE: prefix of token tiles per expert
  int *s_rows = s_tpre + (p.moe ? p.E + 1 : 0);  // [BNT] indexed mode: caller rows of the producer's tile

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;

  // ---- number of valid token tiles (MoE: from the routing offsets) ----
  if (warp == 0) {
    int tvalid = 0;
    if (!p.moe) {
      tvalid = (p.M + BNT - 1) / BNT;
    } else if (p.offsets[p.E] >= 0) {
      int running = 0;
      for (int e0 = 0; e0 < p.E; e0 += 32) {
        const int e = e0 + lane;
        int tiles = 0;
        if (e < p.E) tiles = (p.offsets[e + 1] - p.offsets[e] + BNT - 1) / BNT;
        int incl = tiles;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (e < p.E) s_tpre[e + 1] = running + incl;
        running += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) s_tpre[0] = 0;
      tvalid = running;
    }
    if (tvalid > p.mtiles) tvalid = p.mtiles;  // never beyond the sized workspace
    if (lane == 0) {
      *s_total = (long long)tvalid * p.ntw;  // tiles
      *s_abort = 0;
      *s_last = 0;
    }
  }
  if (tid == 32) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sfree[s], 1 + NDQ);
    }
    for (int a = 0; a < NA; ++a) {
      mbar_init(&afull[a], NDQ);
      mbar_init(&aempty[a], 1);
    }
    for (int d = 0; d < ND; ++d) {
      mbar_init(&accf[d], 1);
      mbar_init(&acce[d], 4);
    }
    fence_barrier_init();
  }
  __syncthreads();
  const Sched sch = make_sched((int)*s_total, p.nctas, p.KB);
  const bool split_mode = !sch.rr && sch.S > 1;
  int t_mine, kb0_mine, kb1_mine, sp_mine;  // first unit of this CTA
  if (!unit_at(sch, cta, p.nctas, p.KB, 0, t_mine, kb0_mine, kb1_mine, sp_mine)) return;

  // tile index -> weight tile, expert, token rows
  auto tile_info = [&](int t) {
    TileInfo ti;
    int slot;
    if (!p.moe && p.group_slots > 1) {
      // dense: token tiles in groups of group_slots, the token tile fastest
      // inside a group, so that the CTAs running together share each weight
      // tile across the group and every weight byte leaves HBM once per group
      const int per = p.group_slots * p.ntw;
      const int grp = t / per;
      const int rem = t - grp * per;
      const int gs = min(p.group_slots, p.mtiles - grp * p.group_slots);
      ti.wt = rem / gs;
      slot = grp * p.group_slots + (rem - ti.wt * gs);
    } else {
      slot = t / p.ntw;
      ti.wt = t - slot * p.ntw;
    }
    if (!p.moe) {
      ti.expert = 0;
      ti.base = slot * BNT;
      ti.nvalid = min(BNT, p.M - ti.base);
    } else {
      int lo = 0, hi = p.E;  // largest e with s_tpre[e] <= slot
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_tpre[mid] <= slot) lo = mid;
        else hi = mid;
      }
      ti.expert = lo;
      ti.base = p.offsets[lo] + (slot - s_tpre[lo]) * BNT;
      ti.nvalid = min(BNT, p.offsets[lo + 1] - ti.base);
    }
    return ti;
  };

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (warp == WARP_PRODUCER) {
    // ================= producer (whole warp in step, lane 0 issues) =================
    const uint64_t pol = p.weights_once ? policy_evict_first() : policy_evict_normal();
    int is = 0;
    bool stop = false;
    for (int u = 0; !stop; ++u) {
      int t, ukb0, ukb1, usp;
      if (!unit_at(sch, cta, p.nctas, p.KB, u, t, ukb0, ukb1, usp)) break;
      const TileInfo ti = tile_info(t);
      if (p.gather) {
        // the tile's caller rows, read once per tile; positions past the
        // valid rows repeat the last one (loaded, never written back)
        for (int i = lane; i < BNT; i += 32) s_rows[i] = p.perm[ti.base + min(i, ti.nvalid - 1)] / p.a_div;
        __syncwarp();
      }
      const int nst = (ukb1 - ukb0 + C::KPS - 1) / C::KPS;
      const int rot = stage_rotation(cta, nst);
      for (int i = 0; i < nst; ++i, ++is) {
      const int kbs = ukb0 + stage_of(i, rot, nst) * C::KPS;
      const int nblk = min(C::KPS, ukb1 - kbs);
      const int s = is % NS;
      if (is >= NS && !mbar_wait(&sfree[s], ((is / NS) - 1) & 1)) { *s_abort = 1; stop = true; break; }
      if (*(volatile int *)s_abort) { stop = true; break; }
      if (lane == 0) {
        const uint8_t *eb = p.packed + (size_t)ti.expert * p.stride;
        uint8_t *st = smem + s * C::STAGE;
        const int g0 = (kbs * TILE_K) >> p.gshift;
        const int g1 = (((kbs + nblk) * TILE_K - 1) >> p.gshift) + 1;
        const uint32_t sb = TR::has_scales ? (uint32_t)((g1 - g0) * BM * TR::sbytes) : 0u;
        const uint32_t zb = TR::has_zero ? (uint32_t)((g1 - g0) * BM) : 0u;
        // indexed mode: ceil(nvalid / 4) gathers of four 128-byte rows per 64-k block
        const uint32_t ab = p.gather ? (uint32_t)(((ti.nvalid + 3) / 4) * 4 * 128) : (uint32_t)C::ACT_KB;
        mbar_arrive_expect_tx(&full[s], ab * nblk + TR::unit * nblk + sb + zb);
        if (!p.gather)
          for (int j = 0; j < nblk; ++j)
            tma_load_2d(st + j * C::ACT_KB, &act_map, (kbs + j) * TILE_K, ti.base, &full[s]);
        bulk_g2s_stream(st + C::ACT, eb + p.w_off + ((size_t)ti.wt * p.KB + kbs) * TR::unit, TR::unit * nblk,
                        &full[s], pol);
        if (TR::has_scales)
          bulk_g2s(st + C::ACT + C::WPK, eb + p.s_off + ((size_t)ti.wt * p.G + g0) * BM * TR::sbytes, sb,
                   &full[s]);
        if (TR::has_zero)
          bulk_g2s(st + C::ACT + C::WPK + C::SC, eb + p.z_off + ((size_t)ti.wt * p.G + g0) * BM, zb, &full[s]);
      }
      __syncwarp();
      if (p.gather) {
        // indexed mode: the stage's 4-row gathers, one group of rows per lane
        // (issued by all lanes at once: from one lane they are ~25 % slower)
        uint8_t *st = smem + s * C::STAGE;
        for (int j = 0; j < nblk; ++j)
          for (int i = 4 * lane; i < ti.nvalid; i += 128)
            tma_gather4(st + j * C::ACT_KB + i * 128, &act_map, (kbs + j) * TILE_K, s_rows[i], s_rows[i + 1],
                        s_rows[i + 2], s_rows[i + 3], &full[s]);
        __syncwarp();
      }
      }
    }
  } else if (warp >= WARP_DQ0) {
    // ================= dequant: thread = weight row =================
    const int dq = warp - WARP_DQ0;       // 0..7
    const int sp = warp & 3;              // TMEM subpartition this warp may access
    const int half = dq >> 2;             // which 32 k of each 64-k block
    const int r = sp * 32 + lane;         // weight row inside the tile
    const uint32_t t_row = tmem + ((uint32_t)(sp * 32) << 16);
    int ia = 0;  // 64-k blocks decoded so far (TMEM A ring position)
    int is = 0;
    bool stop = false;
    for (int u = 0; !stop; ++u) {
      int t, ukb0, ukb1, usp;
      if (!unit_at(sch, cta, p.nctas, p.KB, u, t, ukb0, ukb1, usp)) break;
      const int nst = (ukb1 - ukb0 + C::KPS - 1) / C::KPS;
      const int rot = stage_rotation(cta, nst);
      for (int i = 0; i < nst && !stop; ++i, ++is) {
      const int kbs = ukb0 + stage_of(i, rot, nst) * C::KPS;
      const int nblk = min(C::KPS, ukb1 - kbs);
      const int s = is % NS;
      if (!mbar_wait(&full[s], (is / NS) & 1)) { *s_abort = 1; stop = true; break; }
      const uint8_t *st = smem + s * C::STAGE;
      const uint8_t *sc = st + C::ACT + C::WPK;
      const uint8_t *zp = st + C::ACT + C::WPK + C::SC;
      const int g0 = (kbs * TILE_K) >> p.gshift;
      for (int j = 0; j < nblk; ++j, ++ia) {
        const int a = ia % NA;
        if (ia >= NA && !mbar_wait(&aempty[a], ((ia / NA) - 1) & 1)) { *s_abort = 1; stop = true; break; }
        if (*(volatile int *)s_abort) { stop = true; break; }
        tc_fence_after();
        const int kb = kbs + j;
        const uint8_t *wpk_j = st + C::ACT + j * TR::unit;
        const int gt = ((kb * TILE_K + half * 32) >> p.gshift) - g0;  // group of this thread's first k
        if constexpr (F8) {
          // E4M3 weights go to TMEM unchanged, bytes put back in k order
          uint32_t rg8[8];
  #pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint4 v = *reinterpret_cast<const uint4 *>(wpk_j + (half * 2 + c) * (BM * 16) + r * 16);
            rg8[c * 4 + 0] = __byte_perm(v.x, 0, 0x3120);
            rg8[c * 4 + 1] = __byte_perm(v.y, 0, 0x3120);
            rg8[c * 4 + 2] = __byte_perm(v.z, 0, 0x3120);
            rg8[c * 4 + 3] = __byte_perm(v.w, 0, 0x3120);
          }
          tmem_st8(t_row + (uint32_t)(a * C::A_COLS + half * 8), rg8);
        } else {
          uint32_t rg[16];
          if constexpr (fmt_lowbit(WF)) {
            uint32_t s2, z2;
            lowbit_scale_zero<WF>(sc, zp, gt, r, s2, z2);
            decode_half_lowbit<WF>(wpk_j, s2, z2, r, half, rg);
          } else if constexpr (TR::wbits == 4) {
            const uint4 v = *reinterpret_cast<const uint4 *>(wpk_j + half * (BM * 16) + r * 16);
            const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
            if constexpr (WF == W_INT4 || WF == W_UINT4 || WF == W_MXINT4) {
              // groups are >= 32 k: one scale (and zero point) covers the thread's 32 k
              // (MXINT4: the E8M0 power of two as a bf16, exact)
              const uint32_t s2 = WF == W_MXINT4 ? bcast16(e8m0_code_to_bf16(sc[gt * BM + r]))
                                                 : bcast16(reinterpret_cast<const uint16_t *>(sc)[gt * BM + r]);
              const uint32_t z2 = (WF == W_UINT4) ? bcast16(0x4300u + zp[gt * BM + r]) : 0x43084308u;
  #pragma unroll
              for (int j = 0; j < 4; ++j)
  #pragma unroll
                for (int i = 0; i < 4; ++i)
                  rg[j * 4 + i] = bmul2(bsub2(((w4[j] >> (4 * i)) & 0x000F000Fu) | 0x43004300u, z2), s2);
            } else {
              // MXFP4: one group of 32; NVFP4: two groups of 16 (words 0-1, 2-3)
              uint32_t s2[2];
  #pragma unroll
              for (int q = 0; q < 2; ++q) {
                const uint32_t c = sc[(gt + (WF == W_NVFP4 ? q : 0)) * BM + r];
                s2[q] = bcast16(WF == W_MXFP4 ? e8m0_code_to_bf16(c) : e4m3_code_to_bf16(c));
              }
  #pragma unroll
              for (int j = 0; j < 4; ++j)
  #pragma unroll
                for (int i = 0; i < 4; ++i)
                  rg[j * 4 + i] = bmul2(bmul2(e2m1_pair(w4[j] >> (4 * i)), 0x7E807E80u), s2[j >> 1]);
            }
          } else {
            // 8-bit weights with bf16 activations: two 16-k chunks per thread
  #pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint4 v = *reinterpret_cast<const uint4 *>(wpk_j + (half * 2 + c) * (BM * 16) + r * 16);
              const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  #pragma unroll
              for (int j = 0; j < 4; ++j) {
                rg[c * 8 + j * 2] = bmul2(e4m3_pair(w4[j]), 0x7B807B80u);
                rg[c * 8 + j * 2 + 1] = bmul2(e4m3_pair(w4[j] >> 8), 0x7B807B80u);
              }
            }
          }
          tmem_st16(t_row + (uint32_t)(a * C::A_COLS + half * 16), rg);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[a]);
      }
      if (stop) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sfree[s]);
      }
    }
  } else if (warp == WARP_MMA) {
    // ================= MMA issuer (whole warp in step, lane 0 issues) =================
    constexpr uint32_t idesc = F8 ? idesc_e4m3<BNT>() : idesc_bf16<BNT>();
    int ia = 0;  // 64-k blocks consumed
    int is = 0;
    bool stop = false;
    for (int u = 0; !stop; ++u) {
      int t, ukb0, ukb1, usp;
      if (!unit_at(sch, cta, p.nctas, p.KB, u, t, ukb0, ukb1, usp)) break;
      const int d = u % ND;
      if (u >= ND && !mbar_wait(&acce[d], ((u / ND) - 1) & 1)) { *s_abort = 1; break; }
      const int nst = (ukb1 - ukb0 + C::KPS - 1) / C::KPS;
      const int rot = stage_rotation(cta, nst);
      for (int i = 0; i < nst && !stop; ++i, ++is) {
        const int kbs = ukb0 + stage_of(i, rot, nst) * C::KPS;
        const int nblk = min(C::KPS, ukb1 - kbs);
        const int s = is % NS;
        if (!mbar_wait(&full[s], (is / NS) & 1)) { *s_abort = 1; stop = true; break; }
        for (int j = 0; j < nblk; ++j, ++ia) {
          const int a = ia % NA;
          const bool first = (i == 0 && j == 0);
          const bool last = (i == nst - 1 && j == nblk - 1);
          if (!mbar_wait(&afull[a], (ia / NA) & 1)) { *s_abort = 1; stop = true; break; }
          if (*(volatile int *)s_abort) { stop = true; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t tmem_d = tmem + (uint32_t)(C::D_COL + d * BNT);
            const uint32_t b_addr = smem_u32(smem + s * C::STAGE + j * C::ACT_KB);
            if constexpr (F8) {
              // two K=32 steps of 32 bytes per 64-k block
              const uint64_t bdesc = sw64_desc(b_addr);
#pragma unroll
              for (int k32 = 0; k32 < 2; ++k32)
                mma_ts_f8(tmem_d, tmem + (uint32_t)(a * C::A_COLS + k32 * 8), bdesc + (uint64_t)(k32 * 2), idesc,
                          (!first || k32 > 0) ? 1u : 0u);
            } else {
              const uint64_t bdesc = sw128_desc(b_addr);
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16)
                mma_ts(tmem_d, tmem + (uint32_t)(a * C::A_COLS + k16 * 8), bdesc + (uint64_t)(k16 * 2), idesc,
                       (!first || k16 > 0) ? 1u : 0u);
            }
            mma_commit(&aempty[a]);
            if (last) mma_commit(&accf[d]);
          }
          __syncwarp();
        }
        if (stop) break;
        if (lane == 0) mma_commit(&sfree[s]);
        __syncwarp();
      }
    }
  } else {
    // ================= epilogue: warps 0..3, thread = weight row =================
    const int r = warp * 32 + lane;
    for (int u = 0;; ++u) {
      int t, ukb0, ukb1, usp;
      if (!unit_at(sch, cta, p.nctas, p.KB, u, t, ukb0, ukb1, usp)) break;
      const int d = u % ND;
      const bool ok = mbar_wait(&accf[d], (u / ND) & 1);
      tc_fence_after();
      if (!ok || *(volatile int *)s_abort) break;
      const TileInfo ti = tile_info(t);
      const uint8_t *eb = p.packed + (size_t)ti.expert * p.stride;
      const int n = ti.wt * BM + r;
      float cs = 1.f, gs = 1.f;
      if (WF == W_FP8 && n < p.N) cs = reinterpret_cast<const float *>(eb + p.c_off)[n];
      if (WF == W_NVFP4) gs = reinterpret_cast<const float *>(eb + p.g_off)[0];
      if (p.a_global) gs = __fmul_rn(gs, *p.a_global);
      float *part = p.partial + ((size_t)t * sch.S + usp) * BNT * BM;
      for (int c0 = 0; c0 < BNT && c0 < ti.nvalid; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(C::D_COL + d * BNT + c0), v);
        if (split_mode) {
#pragma unroll
          for (int i = 0; i < 16; ++i) __stcg(&part[(size_t)(c0 + i) * BM + r], v[i]);
        } else {
          // the 16 tokens' output rows (and per-token scales): one load per
          // lane, handed to the other lanes by shuffles
          int orow_l = 0;
          float rs_l = 1.f;
          if (c0 + (lane & 15) < ti.nvalid) {
            const int pos = ti.base + c0 + (lane & 15);
            orow_l = p.moe ? p.perm[pos] : pos;
            if (p.row_scale) rs_l = p.row_scale[p.moe ? orow_l / p.a_div : pos];
          }
          auto stores = [&](auto gated) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int orow = __shfl_sync(0xffffffffu, orow_l, i);
              const float rs = __shfl_sync(0xffffffffu, rs_l, i);
              float x = v[i];
              if (p.row_scale) x *= rs;
              x *= cs;
              x *= gs;
              put_out<decltype(gated)::value>(p, orow, n, x, c0 + i < ti.nvalid && n < p.N);
            }
          };
          if (p.gated) stores(GatedTag<true>{});
          else stores(GatedTag<false>{});
        }
      }
      if (split_mode) __threadfence();  // partial visible before the tile ticket
      // accumulator read: hand it back to the MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[d]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
  }
  if (!split_mode) return;
  // ---- split mode: take the tile's ticket; the last split to arrive sums
  // the S partials in split order (deterministic) with all threads, 16-byte
  // loads and every split's load of an item in flight together.  Every split
  // takes its ticket, so the counter is back at zero once all have arrived.
  if (tid == 0) {
    const int tk = atomicAdd(&p.counters[t_mine], 1);
    const bool last = (tk == sch.S - 1);
    if (last) p.counters[t_mine] = 0;  // ready for the next call
    *s_last = (last && !*(volatile int *)s_abort) ? 1 : 0;
  }
  __syncthreads();
  if (!*(volatile int *)s_last) return;
  __threadfence();
  {
    const TileInfo ti = tile_info(t_mine);
    const uint8_t *eb = p.packed + (size_t)ti.expert * p.stride;
    const float4 *pp = reinterpret_cast<const float4 *>(p.partial + (size_t)t_mine * sch.S * BNT * BM);
    float gs = 1.f;
    if (WF == W_NVFP4) gs = reinterpret_cast<const float *>(eb + p.g_off)[0];
    if (p.a_global) gs = __fmul_rn(gs, *p.a_global);
    for (int item = tid; item < ti.nvalid * (BM / 4); item += THREADS) {
      const int m = item / (BM / 4), r4 = item % (BM / 4);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = 0; s0 < sch.S; s0 += 8) {
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (s0 + j < sch.S) v[j] = __ldcg(pp + ((size_t)(s0 + j) * BNT + m) * (BM / 4) + r4);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (s0 + j < sch.S) {
            acc.x += v[j].x;
            acc.y += v[j].y;
            acc.z += v[j].z;
            acc.w += v[j].w;
          }
      }
      const int pos = ti.base + m;
      const int orow = p.moe ? p.perm[pos] : pos;
      const float rs = p.row_scale ? p.row_scale[p.moe ? orow / p.a_div : pos] : 1.f;
      const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
      float xs[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = ti.wt * BM + r4 * 4 + j;
        xs[j] = 0.f;
        if (n < p.N) {
          float x = a4[j];
          if (p.row_scale) x *= rs;
          if (WF == W_FP8) x *= reinterpret_cast<const float *>(eb + p.c_off)[n];
          x *= gs;
          xs[j] = x;
          if (!p.gated) p.out[(size_t)orow * p.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(x));
        }
      }
      if (p.gated) {
        // the thread's four rows are two gate/up pairs
#pragma unroll
        for (int j = 0; j < 4; j += 2) {
          const int n = ti.wt * BM + r4 * 4 + j;
          if (n < p.N)
            p.out[(size_t)orow * (p.N >> 1) + (n >> 1)] =
                __bfloat16_as_ushort(__float2bfloat16_rn(silu_mul(xs[j], xs[j + 1])));
        }
      }
    }
  }
}

}  // namespace tc

// ---- host side -------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void *ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// [rows, K] row-major activations, box = 64 k x box_rows: bf16 with a
// 128-byte swizzle, or E4M3 bytes with a 64-byte swizzle.
static bool make_act_map(CUtensorMap *m, const void *a, int rows, int K, int box_rows, bool e4m3) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int es = e4m3 ? 1 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * es};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = fn(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void *>(a), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        e4m3 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int sm_count() {
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

// Token tile = the smallest of 16, 32, 64, 128, 256 covering the rows a tile
// is expected to hold.  Up to 32 tokens: the decode kernel, one CTA per SM
// (fewer when there are not 4 k-blocks of work per CTA).  Beyond: two (up to
// 64 tokens) or one CTA per SM of the multi-stage kernel.
TcLaunch plan_tc(int rows_per_tile, int mtiles_bound_moe, int N, int KB, bool moe, int bs) {
  TcLaunch t{};
  t.bnt = rows_per_tile <= 16 ? 16 : rows_per_tile <= 32 ? 32 : rows_per_tile <= 64 ? 64 : rows_per_tile <= 128 ? 128 : 256;
  t.kind = t.bnt <= 32 ? 1 : 0;
  if (bs != BS_NONE) {
    // block-scaled kernel: one CTA per SM, a stage is 1 (FP8), 2 (MX) or 4
    // (NV) 64-k blocks; up to 128 tokens per tile next to the scale columns
    // in tensor memory, 256 without scales (FP8)
    t.kind = 2;
    if (t.bnt > 128 && bs != BS_F8) t.bnt = 128;
    // NVFP4 MoE: about 1.25 x the mean rows per expert, so that the usual
    // spread of rows per expert fits one tile and each expert's weights are
    // read once (measured slower for MXFP4 x MXFP8, whose MMA runs at half
    // the NVFP4 rate)
    if (moe && bs == BS_NV && rows_per_tile > 96 && rows_per_tile <= 160) t.bnt = 192;
    // dense NVFP4 from 1024 rows: 192-token tiles (1.5 x the MMA work per
    // stage for 1.25 x the operand bytes; M = 8192 at N = K = 7168: 383 ->
    // 344 us; at 256 rows the ragged second tile made it slower)
    if (!moe && bs == BS_NV && rows_per_tile >= 1024) t.bnt = 192;
    KB /= (bs == BS_NV ? 4 : bs == BS_MX ? 2 : 1);
  }
  t.ntw = (N + TILE_N - 1) / TILE_N;
  if (t.kind == 2 && t.bnt == 256 && !moe &&
      (long long)t.ntw * ((rows_per_tile + 255) / 256) < 2LL * sm_count()) {
    // fewer than two 256-token tiles per SM: 128-token tiles halve the
    // Stream-K partial sums and split fewer tiles
    t.bnt = 128;
  }
  t.mtiles = moe ? mtiles_bound_moe : (rows_per_tile + t.bnt - 1) / t.bnt;
  if (t.mtiles < 1) t.mtiles = 1;
  const long long iters = (long long)t.ntw * t.mtiles * KB;
  const int sms = sm_count();
  const int slots = t.kind != 0 ? sms : (t.bnt <= 64 ? 2 : 1) * sms;
  long long n = (iters + 3) / 4;
  if (n > slots) n = slots;
  if (n < 1) n = 1;
  t.nctas = (int)n;
  return t;
}

size_t tc_counter_bytes(const TcLaunch &t) {
  const size_t tiles = (size_t)t.ntw * t.mtiles;
  // decode and block-scaled kernels: one ticket per (tile, epilogue warp)
  return align_up(tiles * (t.kind != 0 ? 4 : 1) * sizeof(int), 256);
}

size_t tc_workspace_bytes(const TcLaunch &t) {
  // tile tickets, then the fp32 [bnt][128] partial tiles: one per split
  // (splits <= CTAs), or a head and a tail slot per CTA (Stream-K kernels)
  const size_t parts = t.kind != 0 ? (size_t)t.nctas * 2 : (size_t)t.nctas;
  return tc_counter_bytes(t) + parts * t.bnt * TILE_N * sizeof(float);
}

template <int WF, int BNT, bool F8>
static hq_status tc_launch_one(const CUtensorMap &map, const tc::Params &p, const TcLaunch &t, cudaStream_t st) {
  using C = tc::Cfg<WF, BNT, F8>;
  auto kern = tc::tc_gemm_kernel<WF, BNT, F8>;
  static unsigned configured = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
  if (dev >= 32 || !(configured & (1u << dev))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES) != cudaSuccess)
      return HQ_ERR_CUDA;
    if (dev < 32) configured |= 1u << dev;
  }
  kern<<<t.nctas, tc::THREADS, C::BYTES, st>>>(map, p);
  return check_launch();
}

template <int WF, bool F8 = false>
static hq_status tc_launch_wf(const CUtensorMap &map, const tc::Params &p, const TcLaunch &t, cudaStream_t st) {
  switch (t.bnt) {
    case 16: return tc_launch_one<WF, 16, F8>(map, p, t, st);
    case 32: return tc_launch_one<WF, 32, F8>(map, p, t, st);
    case 64: return tc_launch_one<WF, 64, F8>(map, p, t, st);
    case 128: return tc_launch_one<WF, 128, F8>(map, p, t, st);
    default: return tc_launch_one<WF, 256, F8>(map, p, t, st);
  }
}

hq_status launch_dec_gemm(const Layout &L, const tc::Params &p, const void *a, int a_rows, const TcLaunch &t,
                          cudaStream_t st, bool e4m3_act);

// a_bf16 holds `a_rows` rows of K bf16 values.  Dense and MoE grouped: a tile
// reads the rows [row_base, row_base + BNT) (rows past a tile's end are
// loaded but never written back; rows past the matrix are zero-filled).  MoE
// indexed (gather = 1): a tile gathers the caller rows perm[pos] / a_div.
hq_status launch_tc_gemm(const Layout &L, const void *packed, const void *a_bf16, int a_rows, const float *row_scale,
                         const float *a_global, int M, int moe, int E, const int32_t *offsets, const int32_t *perm,
                         int a_div, int gather, void *out, const TcLaunch &t, void *workspace, cudaStream_t st,
                         bool e4m3_act) {
  if (e4m3_act && L.fmt != W_FP8) return HQ_ERR_UNSUPPORTED;
  CUtensorMap map;
  // indexed mode: one-row boxes for the 4-row gathers
  if (!make_act_map(&map, a_bf16, a_rows, L.K, gather ? 1 : t.bnt, e4m3_act)) return HQ_ERR_CUDA;
  tc::Params p{};
  p.packed = (const uint8_t *)packed;
  p.stride = L.stride;
  p.w_off = L.w_off; p.s_off = L.s_off; p.z_off = L.z_off; p.c_off = L.c_off; p.g_off = L.g_off;
  p.N = L.N; p.K = L.K; p.NT = L.NT; p.KB = L.KB; p.G = L.G; p.group = L.group;
  p.gshift = ((L.group & (L.group - 1)) == 0) ? __builtin_ctz((unsigned)L.group) : 31;
  p.row_scale = row_scale;
  p.a_global = a_global;
  p.gated = L.gated;
  p.M = M;
  p.moe = moe;
  p.E = E;
  p.offsets = offsets;
  p.perm = perm;
  p.a_div = a_div;
  p.gather = gather;
  p.out = (uint16_t *)out;
  p.ntw = t.ntw;
  p.mtiles = t.mtiles;
  p.nctas = t.nctas;
  p.weights_once = (!moe && t.mtiles == 1) ? 1 : 0;
  // raster groups of token tiles whose activations take about 32 MB of L2
  {
    const long long act_tile = (long long)t.bnt * L.K * (e4m3_act ? 1 : 2);
    long long gsl = (32ll << 20) / (act_tile > 0 ? act_tile : 1);
    if (gsl < 1) gsl = 1;
    if (gsl > t.mtiles) gsl = t.mtiles;
    p.group_slots = (int)gsl;
  }
  p.counters = (int *)workspace;
  p.partial = (float *)((uint8_t *)workspace + tc_counter_bytes(t));
  if (t.kind == 1) {
    if (gather && e4m3_act) return HQ_ERR_UNSUPPORTED;
    return launch_dec_gemm(L, p, a_bf16, a_rows, t, st, e4m3_act);
  }
  if (gather && e4m3_act) return HQ_ERR_UNSUPPORTED;
  switch (L.fmt) {
    case W_INT4: return tc_launch_wf<W_INT4>(map, p, t, st);
    case W_E0M3: return tc_launch_wf<W_INT4>(map, p, t, st);  // packed as INT4
    case W_MXINT4: return tc_launch_wf<W_MXINT4>(map, p, t, st);
    case W_INT1: return tc_launch_wf<W_INT1>(map, p, t, st);
    case W_UINT1: return tc_launch_wf<W_UINT1>(map, p, t, st);
    case W_INT2: return tc_launch_wf<W_INT2>(map, p, t, st);
    case W_UINT2: return tc_launch_wf<W_UINT2>(map, p, t, st);
    case W_INT3: return tc_launch_wf<W_INT3>(map, p, t, st);
    case W_UINT3: return tc_launch_wf<W_UINT3>(map, p, t, st);
    case W_E2M3: return tc_launch_wf<W_E2M3>(map, p, t, st);
    case W_E3M2: return tc_launch_wf<W_E3M2>(map, p, t, st);
    case W_UINT4: return tc_launch_wf<W_UINT4>(map, p, t, st);
    case W_MXFP4: return tc_launch_wf<W_MXFP4>(map, p, t, st);
    case W_NVFP4: return tc_launch_wf<W_NVFP4>(map, p, t, st);
    case W_FP8: return e4m3_act ? tc_launch_wf<W_FP8, true>(map, p, t, st) : tc_launch_wf<W_FP8>(map, p, t, st);
    default: return HQ_ERR_UNSUPPORTED;
  }
}

}  // namespace hq
