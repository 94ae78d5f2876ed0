// Tensor-core GEMM with both operands fed straight from TMA: MXFP4 weights x
// MXFP8 activations and NVFP4 weights x NVFP4 activations, with the block
// scales applied by the tensor core itself (no dequantisation anywhere), and
// FP8 weights x per-token FP8 activations.
//
// "Announcing Humming", section "Shared CUDA components across formats and
// architectures": the microscaling formats feed block-scaled MMAs directly on
// hardware that has them; OCP Microscaling Formats (MX) v1.0 specification,
// sections 5.1-5.3 (shared E8M0 scale per 32 elements) and the NVFP4 format
// (E4M3 scale per 16 elements and an FP32 tensor scale).  The sm_100a design:
//
//   * tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale (MX, K = 32 per
//     instruction, E2M1 weights expanded to one byte per code in shared
//     memory by the TMA), kind::mxf4nvf4.block_scale.scale_vec::4X (NV,
//     K = 64, both operands packed E2M1) or kind::f8f6f4 (FP8, K = 32, the
//     per-row and per-token scales in the epilogue); 128 weight rows are
//     operand A, 16..128 tokens operand B (NVFP4 MoE: 192; FP8: up to 256),
//     both in shared memory with a 128-byte swizzle;
//   * the weight codes are stored per 128-row tile in stage chunks, so one
//     stage of a tile is one contiguous piece of HBM (one TMA box);
//   * the scale chunks (128 rows x 4 scales, 512 bytes) go shared memory ->
//     tensor memory with tcgen05.cp.32x128b.warpx4; the weight scales are
//     stored in that order by the repack;
//   * warps: 0..3 epilogue, 4 weight producer (3-D TMA of the codes, bulk copy
//     of the scale chunks), 5 MMA issuer, 6 activation producer (2-D TMA of
//     the codes, bulk copy of the scale chunks);
//   * the activation scales are put in chunk order per token tile by a small
//     kernel first (bs_sf_tiles_kernel; for MoE it also follows the
//     permutation, so the expert-sorted scales are never stored row-wise);
//   * persistent CTAs, one per SM, Stream-K over (tile, stage) iterations with
//     the decode kernel's deterministic last-arriver fixup;
//   * every mbarrier wait is bounded; a timeout records HQ_ERR_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "hq_internal.cuh"

namespace hq {

namespace bs {

using tc::BM;
using tc::Params;
using tc::TileInfo;

constexpr int WARP_W = 4, WARP_MMA = 5, WARP_ACT = 6;
constexpr int THREADS = 7 * 32;
constexpr int TMEM_COLS = 512;

// KIND: BS_MX, BS_NV or BS_F8.  A stage is one 128-byte row of each operand:
// 128 k (MX: E2M1 expanded to bytes / E4M3; F8: E4M3) or 256 k (NV: packed
// E2M1), four MMAs.
template <int KIND, int BNT>
struct Cfg {
  static constexpr int KSTAGE = KIND == BS_NV ? 256 : 128;
  static constexpr int SF_CH = KIND == BS_MX ? 1 : KIND == BS_NV ? 4 : 0;  // scale chunks (4 columns) per stage
  static constexpr int W_SMEM = BM * 128;                  // weight tile in shared memory
  static constexpr int W_GLOBAL = KIND == BS_MX ? BM * 64 : BM * 128;  // packed bytes it is read from
  static constexpr int A_SMEM = BNT * 128;
  static constexpr int SFA_OFF = W_SMEM + A_SMEM;
  // activation scale chunk: 512 bytes per 128 token rows (tiles of more
  // than 128 tokens: a second 512 bytes for rows 128..255)
  static constexpr int SFB_HALVES = BNT > 128 ? 2 : 1;
  static constexpr int SFB_CHB = 512 * SFB_HALVES;  // bytes per activation scale chunk
  static constexpr int SFB_CPC = 4 * SFB_HALVES;    // TMEM columns per activation scale chunk
  static constexpr int SFB_OFF = SFA_OFF + SF_CH * 512;
  static constexpr int STAGE = (SFB_OFF + SF_CH * SFB_CHB + 1023) / 1024 * 1024;
  static constexpr int NS_FIT = (200 * 1024) / STAGE;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int CTRL = 8192;
  static constexpr int BYTES = NS * STAGE + CTRL + 1024;
  static constexpr int ND = 2;
  // TMEM: two accumulators, then the weight and the activation scale columns
  static constexpr int SFA_COL = ND * BNT;
  static constexpr int SFB_COL = SFA_COL + 4 * SF_CH;
  static_assert(SFB_COL + SFB_CPC * SF_CH <= TMEM_COLS, "TMEM budget");
  static_assert(NS >= 3, "stage too large");
};

// Instruction descriptor of the block-scaled kinds (M = 128, K-major A and B);
// FP8: kind::f8f6f4, fp32 accumulator, E4M3 x E4M3.
template <int KIND, int BNT>
__device__ __forceinline__ constexpr uint32_t idesc_bs(uint32_t sf_id) {
  if (KIND == BS_F8) return tc::idesc_e4m3<BNT>();
  return (sf_id << 4)                                            // B scale id (byte of the scale column)
         | ((KIND == BS_MX ? 5u : 1u) << 7)                      // A = E2M1
         | ((KIND == BS_MX ? 0u : 1u) << 10)                     // B = E4M3 (MX) / E2M1 (NV)
         | ((uint32_t)(BNT >> 3) << 17)                          // N
         | ((KIND == BS_MX ? 1u : 0u) << 23)                     // scales: UE8M0 (MX) / UE4M3 (NV)
         | ((uint32_t)(BM >> 4) << 24)                           // M
         | (sf_id << 29);                                        // A scale id
}

// Shared-memory descriptor of a 32-row x 16-byte scale chunk (no swizzle,
// 8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t sf_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(128 >> 4) << 16;
  d |= (uint64_t)(128 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

__device__ __forceinline__ void sf_copy(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

template <int KIND>
__device__ __forceinline__ void mma_bs(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t acc) {
  if constexpr (KIND == BS_F8) {
    (void)sfa;
    (void)sfb;
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc));
  } else if constexpr (KIND == BS_MX) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
            tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb));
  }
}

// 32 fp32 accumulator columns of this warp's TMEM lanes: the load and its
// wait in one statement, so that no use of the registers can be scheduled
// before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Walks a CTA's iterations one stage at a time; a segment is a run inside
// one tile.  Every role walks the same sequence.
struct Walk {
  int t, ks, left;
  bool seg_first, seg_last;
  __device__ __forceinline__ void start(long long beg, long long end, int ki) {
    t = (int)(beg / ki);
    ks = (int)(beg - (long long)t * ki);
    left = (int)(end - beg);
    seg_first = true;
    seg_last = (ks + 1 == ki) || (left == 1);
  }
  __device__ __forceinline__ void next(int ki) {
    --left;
    ++ks;
    seg_first = (ks == ki);
    if (ks == ki) {
      ks = 0;
      ++t;
    }
    seg_last = (ks + 1 == ki) || (left == 1);
  }
};

// The epilogue of one segment, 32 token columns at a time (the accumulator
// columns of a 128-token tile do not fit in registers at once).  Whole tiles
// are written directly; a Stream-K piece is stored as an fp32 partial and the
// last of the CTAs sharing the tile sums the parts in k order.
template <int BNT>
__device__ __forceinline__ void epilogue_segment(const Params &p, const TileInfo &ti, int t, bool whole, bool head,
                                                 uint32_t tacc, uint64_t *acce, float cs, float gs, int cta, int warp,
                                                 int lane, long long total) {
  constexpr int CW = BNT < 32 ? BNT : 32;
  const int r = warp * 32 + lane;
  const int n = ti.wt * BM + r;
  float *part = p.partial + ((size_t)cta * 2 + (head ? 0 : 1)) * BNT * BM;
  auto write = [&](int c0, const float *x) {
    // the chunk's output rows (and FP8 per-token scales): one load per lane,
    // handed to the other lanes by shuffles, so no store waits on a load
    int orow_l = 0;
    float rs_l = 1.f;
    if (c0 + lane < ti.nvalid) {
      const int pos = ti.base + c0 + lane;
      orow_l = p.moe ? p.perm[pos] : pos;
      if (p.row_scale) rs_l = p.row_scale[p.moe ? orow_l / p.a_div : pos];
    }
    auto stores = [&](auto gated) {
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const int orow = __shfl_sync(0xffffffffu, orow_l, i);
        const float rs = __shfl_sync(0xffffffffu, rs_l, i);
        // FP8: per-token x per-row scales; block-scaled kinds: global scales
        float z = x[i];
        if (p.row_scale) z *= rs;
        z *= cs;
        z *= gs;
        tc::put_out<decltype(gated)::value>(p, orow, n, z, c0 + i < ti.nvalid && n < p.N);
      }
    };
    if (p.gated) stores(tc::GatedTag<true>{});
    else stores(tc::GatedTag<false>{});
  };
#pragma unroll 1
  for (int c0 = 0; c0 < BNT; c0 += CW) {
    float v[CW];
    if constexpr (CW == 32) {
      tmem_ld32(tacc + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
    } else {
#pragma unroll
      for (int h = 0; h < CW; h += 16) {
        float v16[16];
        tc::tmem_ld16(tacc + ((uint32_t)(warp * 32) << 16) + (uint32_t)(c0 + h), v16);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[h + i] = v16[i];
      }
    }
    if (whole) {
      write(c0, v);
    } else {
#pragma unroll
      for (int i = 0; i < CW; ++i) __stcg(&part[(size_t)(c0 + i) * BM + r], v[i]);
    }
  }
  // accumulator read: hand it back to the MMA warp
  tc::tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(acce);
  if (whole) return;
  __threadfence();
  __syncwarp();
  const long long t_first = (long long)t * p.KB;
  const int c_first = dec::cta_of(t_first, total, p.nctas);
  const int c_last = dec::cta_of(t_first + p.KB - 1, total, p.nctas);
  int last = 0;
  if (lane == 0) {
    int *ctr = p.counters + (size_t)t * 4 + warp;
    last = (atomicAdd(ctr, 1) == c_last - c_first);
    if (last) *ctr = 0;  // ready for the next call
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
#pragma unroll 1
  for (int c0 = 0; c0 < BNT; c0 += CW) {
    // contributors in k order; the loads of U contributors are in flight together
    constexpr int U = CW <= 16 ? 4 : 2;
    float x[CW];
#pragma unroll
    for (int i = 0; i < CW; ++i) x[i] = 0.f;
    for (int cb = c_first; cb <= c_last; cb += U) {
      float y[U][CW];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = cb + u;
        if (c <= c_last) {
          const float *pc = p.partial + ((size_t)c * 2 + (c == c_first ? 1 : 0)) * BNT * BM + (size_t)c0 * BM + r;
#pragma unroll
          for (int i = 0; i < CW; ++i) y[u][i] = __ldcg(pc + (size_t)i * BM);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (cb + u <= c_last) {
#pragma unroll
          for (int i = 0; i < CW; ++i) x[i] += y[u][i];
        }
    }
    write(c0, x);
  }
}

template <int KIND, int BNT>
__global__ void __launch_bounds__(THREADS, 1)
    bs_gemm_kernel(const __grid_constant__ CUtensorMap w_map, const __grid_constant__ CUtensorMap a_map,
                   const Params p) {
  using C = Cfg<KIND, BNT>;
  constexpr int NS = C::NS, ND = C::ND;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t *ctrl = smem + NS * C::STAGE;
  uint64_t *full = reinterpret_cast<uint64_t *>(ctrl);  // [NS] weights + activations + scales landed
  uint64_t *sfree = full + NS;                           // [NS] stage consumed by the MMAs
  uint64_t *accf = sfree + NS;                           // [ND] accumulator complete
  uint64_t *acce = accf + ND;                            // [ND] accumulator drained
  long long *s_total = reinterpret_cast<long long *>(acce + ND);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(s_total + 1);
  int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);
  int *s_tpre = s_abort + 1;  // [E+1] MoE: prefix of token tiles per expert
  int *s_rows = s_tpre + (p.moe ? p.E + 1 : 0);  // [BNT] indexed mode: caller rows of the producer's tile

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;

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
    if (tvalid > p.mtiles) tvalid = p.mtiles;
    if (lane == 0) {
      *s_total = (long long)tvalid * p.ntw * p.KB;  // (tile, stage) iterations
      *s_abort = 0;
    }
  }
  if (tid == 32) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 2);  // weight producer and activation producer
      mbar_init(&sfree[s], 1);
    }
    for (int d = 0; d < ND; ++d) {
      mbar_init(&accf[d], 1);
      mbar_init(&acce[d], 4);
    }
    fence_barrier_init();
  }
  __syncthreads();
  const long long total = __shfl_sync(0xffffffffu, *s_total, 0);
  const long long beg = dec::range_begin(cta, total, p.nctas);
  const long long end = dec::range_begin(cta + 1, total, p.nctas);
  if (beg >= end) return;

  auto tile_info = [&](int t) {
    TileInfo ti;
    const int slot = t / p.ntw;
    ti.wt = t - slot * p.ntw;
    if (!p.moe) {
      ti.expert = 0;
      ti.base = slot * BNT;
      ti.nvalid = min(BNT, p.M - ti.base);
    } else {
      int lo = 0, hi = p.E;
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

  // The producer warps start loading at once; the warps that use tensor
  // memory wait (named barrier 1) for warp 0's allocation.
  const bool producer = (warp == WARP_W || warp == WARP_ACT);
  uint32_t tmem = 0;
  if (producer) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&w_map) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&a_map) : "memory");
  } else {
    if (warp == 0) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"(TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc::tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"r"(THREADS - 64) : "memory");
    tc::tc_fence_after();
    tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  }
  const int chunks_per_tile = p.K / (4 * p.group);  // scale chunks per 128-row weight tile

  if (warp == WARP_W) {
    // ================= weight producer: codes (3-D TMA) + scale chunks (bulk) =================
    const uint64_t pol = p.weights_once ? policy_evict_first() : policy_evict_normal();
    Walk w;
    w.start(beg, end, p.KB);
    int cur_t = -1, wrow = 0, expert = 0;
    const int nchunk = p.KB;  // stage chunks per weight row (one per stage)
    const uint8_t *sfsrc = nullptr;
    for (int is = 0, s = 0, ph = 0; w.left > 0; ++is, w.next(p.KB)) {
      if (w.t != cur_t) {
        const TileInfo ti = tile_info(w.t);
        expert = ti.expert;
        wrow = ti.wt * nchunk * BM;  // first chunk row of the tile
        sfsrc = p.packed + (size_t)ti.expert * p.stride + p.s_off + (size_t)ti.wt * chunks_per_tile * 512;
        cur_t = w.t;
      }
      if (is >= NS && !mbar_wait(&sfree[s], ph ^ 1)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      if (lane == 0) {
        uint8_t *st = smem + s * C::STAGE;
        // the transaction count of the expanding (MX) copy is the packed bytes read
        mbar_arrive_expect_tx(&full[s], (uint32_t)(C::W_GLOBAL + C::SF_CH * 512));
        // the stage's 128 rows are one contiguous chunk block of the tile
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
            "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(st)),
            "l"(&w_map), "r"(0), "r"(wrow + w.ks * BM), "r"(expert), "r"(smem_u32(&full[s])), "l"(pol)
            : "memory");
        if constexpr (C::SF_CH > 0)
          bulk_g2s(st + C::SFA_OFF, sfsrc + (size_t)w.ks * C::SF_CH * 512, C::SF_CH * 512, &full[s]);
      }
      __syncwarp();
      if (++s == NS) { s = 0; ph ^= 1; }
    }
  } else if (warp == WARP_ACT) {
    // ================= activation producer: codes (2-D TMA, or 4-row gathers =================
    // ================= in MoE indexed mode) + scale chunks (bulk)            =================
    Walk w;
    w.start(beg, end, p.KB);
    int cur_t = -1, base = 0, nvalid = 0;
    const uint8_t *sfsrc = nullptr;
    for (int is = 0, s = 0, ph = 0; w.left > 0; ++is, w.next(p.KB)) {
      if (w.t != cur_t) {
        const TileInfo ti = tile_info(w.t);
        base = ti.base;
        nvalid = ti.nvalid;
        // scale chunks of this tile's token slot, laid out by bs_sf_tiles_kernel
        sfsrc = p.a_sf + (size_t)(w.t / p.ntw) * p.KB * (C::SF_CH * C::SFB_CHB);
        cur_t = w.t;
        if (p.gather) {
          // the tile's caller rows; positions past the valid rows repeat the
          // last one (loaded, never written back)
          for (int i = lane; i < BNT; i += 32) s_rows[i] = p.perm[base + min(i, nvalid - 1)] / p.a_div;
          __syncwarp();
        }
      }
      if (is >= NS && !mbar_wait(&sfree[s], ph ^ 1)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      const int ng = (nvalid + 3) >> 2;  // indexed mode: four 128-byte rows per gather
      if (lane == 0) {
        uint8_t *st = smem + s * C::STAGE;
        if (!p.gather) {
          mbar_arrive_expect_tx(&full[s], (uint32_t)(C::A_SMEM + C::SF_CH * C::SFB_CHB));
          tma_load_2d(st + C::W_SMEM, &a_map, w.ks * 128, base, &full[s]);
        } else {
          mbar_arrive_expect_tx(&full[s], (uint32_t)(ng * 4 * 128 + C::SF_CH * C::SFB_CHB));
        }
        if constexpr (C::SF_CH > 0)
          bulk_g2s(st + C::SFB_OFF, sfsrc + (size_t)w.ks * C::SF_CH * C::SFB_CHB, C::SF_CH * C::SFB_CHB, &full[s]);
      }
      if (p.gather) {
        // the tile's caller rows, one 4-row gather per lane at a time
        __syncwarp();
        uint8_t *st = smem + s * C::STAGE;
        for (int gi = lane; gi < ng; gi += 32)
          tc::tma_gather4(st + C::W_SMEM + gi * 512, &a_map, w.ks * 128, s_rows[4 * gi], s_rows[4 * gi + 1],
                          s_rows[4 * gi + 2], s_rows[4 * gi + 3], &full[s]);
      }
      __syncwarp();
      if (++s == NS) { s = 0; ph ^= 1; }
    }
  } else if (warp == WARP_MMA) {
    // ================= MMA issuer (one elected lane) =================
    Walk w;
    w.start(beg, end, p.KB);
    int q = 0, d = 0, dph = 0;
    for (int is = 0, s = 0, ph = 0; w.left > 0; ++is, w.next(p.KB)) {
      if (w.seg_first) {
        if (q > 0 && ++d == ND) { d = 0; dph ^= 1; }
        if (q >= ND && !mbar_wait(&acce[d], dph ^ 1)) { *s_abort = 1; break; }
        ++q;
      }
      if (!mbar_wait(&full[s], ph)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      tc::tc_fence_after();
      const uint32_t st = smem_u32(smem + s * C::STAGE);
      const uint64_t adesc = tc::sw128_desc(st);
      const uint64_t bdesc = tc::sw128_desc(st + C::W_SMEM);
      const uint32_t tmem_d = tmem + (uint32_t)(d * BNT);
      const uint32_t acc0 = w.seg_first ? 0u : 1u;
      if (dec::elect_one()) {
        // scale chunks -> TMEM; the copies and the MMAs below execute in issue
        // order, so the previous stage's MMAs have read the old scales
#pragma unroll
        for (int c = 0; c < C::SF_CH; ++c) {
          sf_copy(tmem + (uint32_t)(C::SFA_COL + 4 * c), sf_desc(st + C::SFA_OFF + c * 512));
#pragma unroll
          for (int h = 0; h < C::SFB_HALVES; ++h)
            sf_copy(tmem + (uint32_t)(C::SFB_COL + C::SFB_CPC * c + 4 * h),
                    sf_desc(st + C::SFB_OFF + c * C::SFB_CHB + h * 512));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          // MX: one scale per 32 k = byte j of the chunk's column; NV: chunk j, all 4 bytes
          const uint32_t sf_id = KIND == BS_MX ? (uint32_t)j : 0u;
          const uint32_t cola = KIND == BS_MX ? 0u : (uint32_t)(4 * j);
          const uint32_t colb = KIND == BS_MX ? 0u : (uint32_t)(C::SFB_CPC * j);
          mma_bs<KIND>(tmem_d, adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc_bs<KIND, BNT>(sf_id),
                       (tmem + C::SFA_COL + cola) | (sf_id << 30), (tmem + C::SFB_COL + colb) | (sf_id << 30),
                       j > 0 ? 1u : acc0);
        }
        tc::mma_commit(&sfree[s]);
        if (w.seg_last) tc::mma_commit(&accf[d]);
      }
      __syncwarp();
      if (++s == NS) { s = 0; ph ^= 1; }
    }
  } else if (warp < 4) {
    // ================= epilogue: warps 0..3, thread = weight row =================
    int t = (int)(beg / p.KB);
    int ks0 = (int)(beg - (long long)t * p.KB);
    int left = (int)(end - beg);
    for (int d = 0, dph = 0; left > 0;) {
      const int seg_len = min(p.KB - ks0, left);
      const bool whole = (ks0 == 0) && (seg_len == p.KB);
      const bool ok = mbar_wait(&accf[d], dph);
      tc::tc_fence_after();
      if (!ok || *(volatile int *)s_abort) break;
      const TileInfo ti = tile_info(t);
      const uint8_t *eb = p.packed + (size_t)ti.expert * p.stride;
      float cs = 1.f, gs = 1.f;
      if (KIND == BS_NV) {
        gs = reinterpret_cast<const float *>(eb + p.g_off)[0];
        if (p.a_global) gs = __fmul_rn(gs, *p.a_global);
      }
      if (KIND == BS_F8) cs = reinterpret_cast<const float *>(eb + p.c_off)[ti.wt * BM + warp * 32 + lane];
      epilogue_segment<BNT>(p, ti, t, whole, ks0 > 0, tmem + (uint32_t)(d * BNT), &acce[d], cs, gs, cta, warp, lane,
                            total);
      left -= seg_len;
      ++t;
      ks0 = 0;
      if (++d == ND) { d = 0; dph ^= 1; }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

// Activation scales in the order the block-scaled kernel copies them: for
// token slot q, stage ks and chunk c, 512 bytes per 128 rows (1024 for tiles
// of more than 128 tokens, rows 128..255 in the second half) with 4 scales of
// each row n at (n % 32) * 16 + (n / 32 % 4) * 4 of its half (rows past the
// slot's valid rows, and n >= bnt, are zero).  Dense: slot q = rows [q * bnt, q * bnt +
// bnt) of the activations.  MoE: slots enumerate the experts' token tiles in
// expert order (rows offsets[e] + i * bnt, ...) and expert-sorted row r reads
// caller row perm[r] / div.  One thread per 4-byte word.
__global__ void bs_sf_tiles_kernel(int slots, int bnt, int kst, int sf_ch, int ld, const uint8_t *__restrict__ sf,
                                   int M, int moe, int E, const int32_t *__restrict__ offsets,
                                   const int32_t *__restrict__ perm, int div, uint32_t *__restrict__ out) {
  extern __shared__ int tpre[];  // [E + 1] MoE: prefix of token tiles per expert
  bool routed_ok = true;
  if (moe) {
    routed_ok = offsets[E] >= 0;
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      int running = 0;
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        int tiles = 0;
        if (e < E && routed_ok) tiles = (offsets[e + 1] - offsets[e] + bnt - 1) / bnt;
        int incl = tiles;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (e < E) tpre[e + 1] = running + incl;
        running += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) tpre[0] = 0;
    }
    __syncthreads();
  }
  const int rows = bnt > 128 ? 256 : 128;  // token rows per chunk (512 bytes per 128)
  const size_t total = (size_t)slots * kst * sf_ch * rows;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(idx % rows);
    const size_t rest = idx / rows;
    const int c = (int)(rest % sf_ch);
    const size_t rest2 = rest / sf_ch;
    const int ks = (int)(rest2 % kst);
    const int q = (int)(rest2 / kst);
    uint32_t v = 0;
    if (n < bnt) {
      int src = -1;
      if (!moe) {
        const int row = q * bnt + n;
        if (row < M) src = row;
      } else if (routed_ok && q < tpre[E]) {
        int lo = 0, hi = E;  // largest e with tpre[e] <= q
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (tpre[mid] <= q) lo = mid;
          else hi = mid;
        }
        const int row = offsets[lo] + (q - tpre[lo]) * bnt + n;
        if (row < offsets[lo + 1]) src = perm[row] / div;
      }
      if (src >= 0) v = *reinterpret_cast<const uint32_t *>(sf + (size_t)src * ld + ((size_t)ks * sf_ch + c) * 4);
    }
    out[(((size_t)q * kst + ks) * sf_ch + c) * rows + (n >> 7) * 128 + (n & 31) * 4 + ((n & 127) >> 5)] = v;
  }
}


// ---- FP8 with 128 x 128 block weight scales and per-(token, 128 k) activation
// scales.  The tensor core cannot apply arbitrary fp32 block scales, so each
// 128-k stage is multiplied into its own TMEM accumulator (a ring of NP) and
// the epilogue warps promote it into fp32 registers:
//     acc[m] += P[m] * (s_w[tile, stage] * s_a[m, stage]),
// the product summed per stage in the tensor core's fp32 and the stages in
// k order.  Warps: 0..3 promotion + output (thread = weight row, BNT
// accumulators in registers), 4 weight producer, 5 MMA issuer, 6 activation
// producer (codes by TMA or, indexed mode, cp.async gathers; the stage's
// activation scales by a bulk copy from their per-token-tile relayout).
template <int BNT>
struct CfgF8B {
  static constexpr int W_SMEM = BM * 128;
  static constexpr int A_SMEM = BNT * 128;
  static constexpr int SA_OFF = W_SMEM + A_SMEM;
  static constexpr int STAGE = (SA_OFF + BNT * 4 + 1023) / 1024 * 1024;
  static constexpr int NS_FIT = (200 * 1024) / STAGE;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int CTRL = 8192;
  static constexpr int BYTES = NS * STAGE + CTRL + 1024;
  static constexpr int NP = (512 / BNT) > 4 ? 4 : (512 / BNT);  // stage accumulators in TMEM
  static constexpr int TMEM_COLS = NP * BNT < 32 ? 32 : NP * BNT;
  // promotion groups of four warps (one per TMEM lane quadrant), each taking
  // BNT / PG token columns of every stage: warps 0..3 and, with two groups,
  // warps 7..10 (after the producers and the MMA issuer)
  static constexpr int PG = BNT >= 64 ? 2 : 1;
  static constexpr int PCOLS = BNT / PG;
  static constexpr int THREADS = (7 + 4 * (PG - 1)) * 32;
  static_assert(NS >= 3 && NP >= 2, "budget");
  static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0, "TMEM allocation is a power of two");
};

// Output of one promoted segment (thread = weight row n): whole tiles are
// written; a Stream-K piece is stored as fp32 partials, and the last of the
// CTAs sharing the tile sums the parts in k order (32 columns at a time).
template <int BNT, int PG>
__device__ __forceinline__ void f8b_finish(const Params &p, const TileInfo &ti, int t, bool whole, bool head,
                                           const float (&acc)[BNT / PG], int cbeg, int cta, int quad, int lane,
                                           long long total) {
  constexpr int PCOLS = BNT / PG;
  constexpr int CW = BNT < 32 ? BNT : 32;
  constexpr int CWP = PCOLS < 32 ? PCOLS : 32;
  const int r = quad * 32 + lane;
  const int n = ti.wt * BM + r;
  auto write = [&](int c0, const float *x) {
    int orow_l = 0;
    if (c0 + lane < ti.nvalid) {
      const int pos = ti.base + c0 + lane;
      orow_l = p.moe ? p.perm[pos] : pos;
    }
    auto stores = [&](auto gated) {
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const int orow = __shfl_sync(0xffffffffu, orow_l, i);
        tc::put_out<decltype(gated)::value>(p, orow, n, x[i], c0 + i < ti.nvalid && n < p.N);
      }
    };
    if (p.gated) stores(tc::GatedTag<true>{});
    else stores(tc::GatedTag<false>{});
  };
  if (whole) {
    // this group's columns [cbeg, cbeg + PCOLS)
    static_assert(CWP == CW, "a group writes whole column chunks");
#pragma unroll
    for (int c0 = 0; c0 < PCOLS; c0 += CW) write(cbeg + c0, acc + c0);
    return;
  }
  float *part = p.partial + ((size_t)cta * 2 + (head ? 0 : 1)) * BNT * BM;
#pragma unroll
  for (int m = 0; m < PCOLS; ++m) __stcg(&part[(size_t)(cbeg + m) * BM + r], acc[m]);
  __threadfence();
  __syncwarp();
  const long long t_first = (long long)t * p.KB;
  const int c_first = dec::cta_of(t_first, total, p.nctas);
  const int c_last = dec::cta_of(t_first + p.KB - 1, total, p.nctas);
  int last = 0;
  if (lane == 0) {
    // one ticket per lane quadrant: every group of every contributing CTA
    // takes one; the last sums all BNT columns of the quadrant's rows
    int *ctr = p.counters + (size_t)t * 4 + quad;
    last = (atomicAdd(ctr, 1) == PG * (c_last - c_first + 1) - 1);
    if (last) *ctr = 0;  // ready for the next call
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
#pragma unroll 1
  for (int c0 = 0; c0 < BNT; c0 += CW) {
    float x[CW];
#pragma unroll
    for (int i = 0; i < CW; ++i) x[i] = 0.f;
    for (int c = c_first; c <= c_last; ++c) {
      const float *pc = p.partial + ((size_t)c * 2 + (c == c_first ? 1 : 0)) * BNT * BM + (size_t)c0 * BM + r;
#pragma unroll
      for (int i = 0; i < CW; ++i) x[i] += __ldcg(pc + (size_t)i * BM);
    }
    write(c0, x);
  }
}

template <int BNT>
__global__ void __launch_bounds__(CfgF8B<BNT>::THREADS, 1)
    bsf_gemm_kernel(const __grid_constant__ CUtensorMap w_map, const __grid_constant__ CUtensorMap a_map,
                    const Params p) {
  using C = CfgF8B<BNT>;
  constexpr int NS = C::NS, NP = C::NP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t *ctrl = smem + NS * C::STAGE;
  uint64_t *full = reinterpret_cast<uint64_t *>(ctrl);  // [NS] codes + activation scales landed
  uint64_t *sfree = full + NS;                           // [NS] MMAs done and the stage's scales read
  uint64_t *pfull = sfree + NS;                          // [NP] stage accumulator complete
  uint64_t *pempty = pfull + NP;                         // [NP] stage accumulator promoted
  long long *s_total = reinterpret_cast<long long *>(pempty + NP);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(s_total + 1);
  int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);
  int *s_tpre = s_abort + 1;                      // [E+1] MoE: prefix of token tiles per expert
  int *s_rows = s_tpre + (p.moe ? p.E + 1 : 0);  // [BNT] indexed mode: caller rows of the producer's tile

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cta = blockIdx.x;
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
    if (tvalid > p.mtiles) tvalid = p.mtiles;
    if (lane == 0) {
      *s_total = (long long)tvalid * p.ntw * p.KB;  // (tile, stage) iterations
      *s_abort = 0;
    }
  }
  if (tid == 32) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 2);      // weight producer and activation producer
      mbar_init(&sfree[s], 1 + 4 * C::PG);  // MMA commit and the promotion warps
    }
    for (int q = 0; q < NP; ++q) {
      mbar_init(&pfull[q], 1);
      mbar_init(&pempty[q], 4 * C::PG);
    }
    fence_barrier_init();
  }
  __syncthreads();
  const long long total = __shfl_sync(0xffffffffu, *s_total, 0);
  const long long beg = dec::range_begin(cta, total, p.nctas);
  const long long end = dec::range_begin(cta + 1, total, p.nctas);
  if (beg >= end) return;

  auto tile_info = [&](int t) {
    TileInfo ti;
    const int slot = t / p.ntw;
    ti.wt = t - slot * p.ntw;
    if (!p.moe) {
      ti.expert = 0;
      ti.base = slot * BNT;
      ti.nvalid = min(BNT, p.M - ti.base);
    } else {
      int lo = 0, hi = p.E;
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

  const bool producer = (warp == WARP_W || warp == WARP_ACT);
  uint32_t tmem = 0;
  if (producer) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&w_map) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&a_map) : "memory");
  } else {
    if (warp == 0) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"(C::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc::tc_fence_before();
    asm volatile("bar.sync 1, %0;" ::"r"(C::THREADS - 64) : "memory");
    tc::tc_fence_after();
    tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  }

  if (warp == WARP_W) {
    // ================= weight producer: one 3-D TMA of the stage's codes =================
    const uint64_t pol = p.weights_once ? policy_evict_first() : policy_evict_normal();
    Walk w;
    w.start(beg, end, p.KB);
    int cur_t = -1, wrow = 0, expert = 0;
    for (int is = 0, s = 0, ph = 0; w.left > 0; ++is, w.next(p.KB)) {
      if (w.t != cur_t) {
        const TileInfo ti = tile_info(w.t);
        expert = ti.expert;
        wrow = ti.wt * p.KB * BM;
        cur_t = w.t;
      }
      if (is >= NS && !mbar_wait(&sfree[s], ph ^ 1)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      if (lane == 0) {
        uint8_t *st = smem + s * C::STAGE;
        mbar_arrive_expect_tx(&full[s], (uint32_t)C::W_SMEM);
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
            "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(st)),
            "l"(&w_map), "r"(0), "r"(wrow + w.ks * BM), "r"(expert), "r"(smem_u32(&full[s])), "l"(pol)
            : "memory");
      }
      __syncwarp();
      if (++s == NS) { s = 0; ph ^= 1; }
    }
  } else if (warp == WARP_ACT) {
    // ================= activation producer: codes + the stage's scales =================
    Walk w;
    w.start(beg, end, p.KB);
    int cur_t = -1, base = 0, nvalid = 0;
    const uint8_t *sasrc = nullptr;
    for (int is = 0, s = 0, ph = 0; w.left > 0; ++is, w.next(p.KB)) {
      if (w.t != cur_t) {
        const TileInfo ti = tile_info(w.t);
        base = ti.base;
        nvalid = ti.nvalid;
        // activation scales of this tile's token slot: [KB][BNT] fp32
        sasrc = p.a_sf + (size_t)(w.t / p.ntw) * p.KB * BNT * 4;
        cur_t = w.t;
        if (p.gather) {
          for (int i = lane; i < BNT; i += 32) s_rows[i] = p.perm[base + min(i, nvalid - 1)] / p.a_div;
          __syncwarp();
        }
      }
      if (is >= NS && !mbar_wait(&sfree[s], ph ^ 1)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      uint8_t *st = smem + s * C::STAGE;
      const int ng = (nvalid + 3) >> 2;  // indexed mode: four 128-byte rows per gather
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], (uint32_t)((p.gather ? ng * 4 * 128 : C::A_SMEM) + BNT * 4));
        if (!p.gather) tma_load_2d(st + C::W_SMEM, &a_map, w.ks * 128, base, &full[s]);
        bulk_g2s(st + C::SA_OFF, sasrc + (size_t)w.ks * BNT * 4, (uint32_t)(BNT * 4), &full[s]);
      }
      if (p.gather) {
        // one 4-row gather per lane at a time
        __syncwarp();
        for (int gi = lane; gi < ng; gi += 32)
          tc::tma_gather4(st + C::W_SMEM + gi * 512, &a_map, w.ks * 128, s_rows[4 * gi], s_rows[4 * gi + 1],
                          s_rows[4 * gi + 2], s_rows[4 * gi + 3], &full[s]);
      }
      __syncwarp();
      if (++s == NS) { s = 0; ph ^= 1; }
    }
  } else if (warp == WARP_MMA) {
    // ================= MMA issuer: each stage into its own accumulator =================
    constexpr uint32_t idesc = tc::idesc_e4m3<BNT>();
    Walk w;
    w.start(beg, end, p.KB);
    for (int is = 0, s = 0, ph = 0, q = 0, qph = 0; w.left > 0; ++is, w.next(p.KB)) {
      if (!mbar_wait(&full[s], ph)) { *s_abort = 1; break; }
      if (is >= NP && !mbar_wait(&pempty[q], qph ^ 1)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      tc::tc_fence_after();
      const uint32_t st = smem_u32(smem + s * C::STAGE);
      const uint64_t adesc = tc::sw128_desc(st);
      const uint64_t bdesc = tc::sw128_desc(st + C::W_SMEM);
      if (dec::elect_one()) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_bs<BS_F8>(tmem + (uint32_t)(q * BNT), adesc + (uint64_t)(2 * j), bdesc + (uint64_t)(2 * j), idesc, 0u,
                        0u, j > 0 ? 1u : 0u);
        tc::mma_commit(&pfull[q]);
        tc::mma_commit(&sfree[s]);
      }
      __syncwarp();
      if (++s == NS) { s = 0; ph ^= 1; }
      if (++q == NP) { q = 0; qph ^= 1; }
    }
  } else if (warp < 4 || warp >= 7) {
    // ================= promotion: thread = weight row of lane quadrant warp & 3, =================
    // ================= token columns [cb, cb + PCOLS) (group 0: warps 0..3, 1: 7..10) =================
    constexpr int PCOLS = C::PCOLS;
    const int quad = warp & 3;
    const int cb = warp >= 7 ? PCOLS : 0;
    float acc[PCOLS];
    Walk w;
    w.start(beg, end, p.KB);
    int t0 = w.t, ks0 = w.ks;  // where the current segment started
    // the weight block scale of a stage, loaded one stage ahead so that its
    // latency is off the promotion's path (tile lookups only when the tile changes)
    int sw_t = -1;
    const float *sw_row = nullptr;
    auto sw_of = [&](int t, int ks) {
      if (t != sw_t) {
        const TileInfo ti = tile_info(t);
        sw_row = reinterpret_cast<const float *>(p.packed + (size_t)ti.expert * p.stride + p.c_off) +
                 (size_t)ti.wt * p.KB;
        sw_t = t;
      }
      return __ldg(sw_row + ks);
    };
    float sw_next = sw_of(w.t, w.ks);
    for (int is = 0, s = 0, ph = 0, q = 0, qph = 0; w.left > 0; ++is, w.next(p.KB)) {
      if (w.seg_first) {
#pragma unroll
        for (int m = 0; m < PCOLS; ++m) acc[m] = 0.f;
        t0 = w.t;
        ks0 = w.ks;
      }
      const float sw = sw_next;
      if (w.left > 1) {
        Walk wn = w;
        wn.next(p.KB);
        sw_next = sw_of(wn.t, wn.ks);
      }
      // the stage (its activation scales) has landed, and its MMAs are done
      const bool ok = mbar_wait(&full[s], ph) && mbar_wait(&pfull[q], qph);
      tc::tc_fence_after();
      if (!ok || *(volatile int *)s_abort) break;
      const float *sa = reinterpret_cast<const float *>(smem + s * C::STAGE + C::SA_OFF);
      constexpr int CL = PCOLS < 32 ? 16 : 32;  // columns per TMEM load (one wait each)
      const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(q * BNT + cb);
#pragma unroll
      for (int c0 = 0; c0 < PCOLS; c0 += CL) {
        float v[CL];
        if constexpr (CL == 32) tmem_ld32(tq + (uint32_t)c0, v);
        else tc::tmem_ld16(tq + (uint32_t)c0, v);
#pragma unroll
        for (int i = 0; i < CL; i += 4) {
          const float4 a4 = *reinterpret_cast<const float4 *>(sa + cb + c0 + i);
          acc[c0 + i] = fmaf(v[i], __fmul_rn(sw, a4.x), acc[c0 + i]);
          acc[c0 + i + 1] = fmaf(v[i + 1], __fmul_rn(sw, a4.y), acc[c0 + i + 1]);
          acc[c0 + i + 2] = fmaf(v[i + 2], __fmul_rn(sw, a4.z), acc[c0 + i + 2]);
          acc[c0 + i + 3] = fmaf(v[i + 3], __fmul_rn(sw, a4.w), acc[c0 + i + 3]);
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&pempty[q]);
        mbar_arrive(&sfree[s]);
      }
      if (w.seg_last) {
        const bool whole = (ks0 == 0) && (w.ks == p.KB - 1);
        f8b_finish<BNT, C::PG>(p, tile_info(t0), t0, whole, ks0 > 0, acc, cb, cta, quad, lane, total);
      }
      if (++s == NS) { s = 0; ph ^= 1; }
      if (++q == NP) { q = 0; qph ^= 1; }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
  }
}

// Activation scales per token tile for the block-scaled FP8 kernel: out
// [slots][kst][bnt] fp32 with out[q][ks][n] = the scale of the tile's row n
// for stage ks (0 past the slot's valid rows).  Dense: slot q = rows
// [q * bnt, q * bnt + bnt); MoE: as bs_sf_tiles_kernel, expert-sorted row r
// reads caller row perm[r] / div.  One thread per output value.
__global__ void f8b_sa_tiles_kernel(int slots, int bnt, int kst, const float *__restrict__ sa, int M, int moe, int E,
                                    const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm, int div,
                                    float *__restrict__ out) {
  extern __shared__ int tpre[];
  bool routed_ok = true;
  if (moe) {
    routed_ok = offsets[E] >= 0;
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      int running = 0;
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        int tiles = 0;
        if (e < E && routed_ok) tiles = (offsets[e + 1] - offsets[e] + bnt - 1) / bnt;
        int incl = tiles;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        if (e < E) tpre[e + 1] = running + incl;
        running += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) tpre[0] = 0;
    }
    __syncthreads();
  }
  const size_t total = (size_t)slots * kst * bnt;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int n = (int)(idx % bnt);
    const size_t rest = idx / bnt;
    const int ks = (int)(rest % kst);
    const int q = (int)(rest / kst);
    int src = -1;
    if (!moe) {
      const int row = q * bnt + n;
      if (row < M) src = row;
    } else if (routed_ok && q < tpre[E]) {
      int lo = 0, hi = E;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tpre[mid] <= q) lo = mid;
        else hi = mid;
      }
      const int row = offsets[lo] + (q - tpre[lo]) * bnt + n;
      if (row < offsets[lo + 1]) src = perm[row] / div;
    }
    out[idx] = src >= 0 ? sa[(size_t)src * kst + ks] : 0.f;
  }
}

}  // namespace bs

// ---- host side -------------------------------------------------------------------

// Weight codes of all experts as rows of one stage chunk ([NT][stages][128]
// rows per expert), experts `stride` bytes apart.  MX: 4-bit elements
// expanded to one byte each in shared memory (box 128 codes x 128 rows); NV,
// F8: bytes (box 128 bytes x 128 rows).
static bool make_bs_weight_map(CUtensorMap *m, const Layout &L, const void *packed, int E) {
  auto fn = encode_fn();
  if (!fn) return false;
  const bool mx = L.bs == BS_MX;
  const size_t cb = (size_t)L.bs_chunk_bytes();
  const size_t rows = (size_t)L.NT * (L.bs_row_bytes() / cb) * TILE_N;
  cuuint64_t dims[3] = {(cuuint64_t)(mx ? 2 * cb : cb), (cuuint64_t)rows, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)cb, (cuuint64_t)L.stride};
  cuuint32_t box[3] = {128u, 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(m, mx ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                        const_cast<uint8_t *>((const uint8_t *)packed + L.w_off), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Activation codes [rows][row_bytes] (E4M3 bytes or packed E2M1), box 128 bytes x bnt rows.
static bool make_bs_act_map(CUtensorMap *m, const void *a, int rows, int row_bytes, int bnt) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {128u, (cuuint32_t)bnt};
  cuuint32_t estr[2] = {1u, 1u};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(a), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int KIND, int BNT>
static hq_status bs_launch_one(const CUtensorMap &wm, const CUtensorMap &am, const tc::Params &p, const TcLaunch &t,
                               cudaStream_t st) {
  using C = bs::Cfg<KIND, BNT>;
  auto kern = bs::bs_gemm_kernel<KIND, BNT>;
  static unsigned configured = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
  if (dev >= 32 || !(configured & (1u << dev))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES) != cudaSuccess)
      return HQ_ERR_CUDA;
    if (dev < 32) configured |= 1u << dev;
  }
  kern<<<t.nctas, bs::THREADS, C::BYTES, st>>>(wm, am, p);
  return check_launch();
}

template <int BNT>
static hq_status bsf_launch_one(const CUtensorMap &wm, const CUtensorMap &am, const tc::Params &p, const TcLaunch &t,
                                cudaStream_t st) {
  using C = bs::CfgF8B<BNT>;
  auto kern = bs::bsf_gemm_kernel<BNT>;
  static unsigned configured = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
  if (dev >= 32 || !(configured & (1u << dev))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES) != cudaSuccess)
      return HQ_ERR_CUDA;
    if (dev < 32) configured |= 1u << dev;
  }
  kern<<<t.nctas, C::THREADS, C::BYTES, st>>>(wm, am, p);
  return check_launch();
}

template <int KIND>
static hq_status bs_launch_kind(const CUtensorMap &wm, const CUtensorMap &am, const tc::Params &p,
                                const TcLaunch &t, cudaStream_t st) {
  switch (t.bnt) {
    case 16: return bs_launch_one<KIND, 16>(wm, am, p, t, st);
    case 32: return bs_launch_one<KIND, 32>(wm, am, p, t, st);
    case 64: return bs_launch_one<KIND, 64>(wm, am, p, t, st);
    case 128: return bs_launch_one<KIND, 128>(wm, am, p, t, st);
    case 192:
      if constexpr (KIND == BS_NV) return bs_launch_one<KIND, 192>(wm, am, p, t, st);
      return HQ_ERR_UNSUPPORTED;
    default:
      if constexpr (KIND == BS_F8) return bs_launch_one<KIND, 256>(wm, am, p, t, st);
      return HQ_ERR_UNSUPPORTED;
  }
}

size_t bs_sf_tiles_bytes(const Layout &L, const TcLaunch &t) {
  if (L.bs == BS_NONE || L.bs == BS_F8) return 0;
  if (L.bs == BS_F8B) return (size_t)t.mtiles * (L.K / 128) * t.bnt * 4;
  const int kstage = L.bs == BS_MX ? 128 : 256;
  const int sf_ch = L.bs == BS_MX ? 1 : 4;
  return (size_t)t.mtiles * (L.K / kstage) * sf_ch * (t.bnt > 128 ? 1024 : 512);
}

// a_codes: `a_rows` activation rows (MXFP8, FP8: K E4M3 bytes per row; NVFP4:
// K/2 packed bytes) in the order the tiles read them: dense rows of a, or MoE
// expert-sorted rows; with `gather` (MoE indexed mode) the caller's rows,
// expert-sorted row r read from row perm[r] / a_div.  a_scales: the caller's scale rows (MXFP8: K/32 E8M0,
// NVFP4: K/16 UE4M3, FP8: one fp32 per row), read through perm / div for MoE.
// Outputs go to row perm[r] for MoE.  sf_tiles: bs_sf_tiles_bytes() of
// scratch (none for FP8).
hq_status launch_bs_gemm(const Layout &L, const void *packed, int E, const void *a_codes, int a_rows,
                         const void *a_scales, int a_div, const float *a_global, int M, int moe,
                         const int32_t *offsets, const int32_t *perm, void *out, const TcLaunch &t,
                         void *workspace, void *sf_tiles, cudaStream_t st, int gather) {
  if (L.bs == BS_NONE || t.kind != 2) return HQ_ERR_UNSUPPORTED;
  if (((uintptr_t)packed & 31) != 0 || ((uintptr_t)a_scales & 3) != 0) return HQ_ERR_INVALID_ARG;
  const int kstage = L.bs == BS_NV ? 256 : 128;
  const int sf_ch = L.bs == BS_MX ? 1 : 4;
  const int row_bytes = L.bs == BS_NV ? L.K / 2 : L.K;
  CUtensorMap wm, am;
  if (!make_bs_weight_map(&wm, L, packed, E)) return HQ_ERR_CUDA;
  // indexed mode: one-row boxes for the 4-row gathers of caller rows
  if (!make_bs_act_map(&am, a_codes, a_rows, row_bytes, gather ? 1 : t.bnt)) return HQ_ERR_CUDA;
  if (L.bs == BS_F8B) {
    // activation scales per token tile and stage: [mtiles][K / 128][bnt] fp32
    const size_t n = (size_t)t.mtiles * (L.K / 128) * t.bnt;
    size_t blocks = (n + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    bs::f8b_sa_tiles_kernel<<<(int)blocks, 256, moe ? (E + 1) * sizeof(int) : 0, st>>>(
        t.mtiles, t.bnt, L.K / 128, (const float *)a_scales, M, moe, E, offsets, perm, a_div, (float *)sf_tiles);
    const hq_status s = check_launch();
    if (s != HQ_OK) return s;
  } else if (L.bs != BS_F8) {
    const size_t words = (size_t)t.mtiles * (L.K / kstage) * sf_ch * (t.bnt > 128 ? 256 : 128);
    size_t blocks = (words + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    bs::bs_sf_tiles_kernel<<<(int)blocks, 256, moe ? (E + 1) * sizeof(int) : 0, st>>>(
        t.mtiles, t.bnt, L.K / kstage, sf_ch, L.K / L.group, (const uint8_t *)a_scales, M, moe, E, offsets, perm,
        a_div, (uint32_t *)sf_tiles);
    const hq_status s = check_launch();
    if (s != HQ_OK) return s;
  }
  tc::Params p{};
  p.packed = (const uint8_t *)packed;
  p.stride = L.stride;
  p.w_off = L.w_off; p.s_off = L.s_off; p.z_off = L.z_off; p.c_off = L.c_off; p.g_off = L.g_off;
  p.N = L.N; p.K = L.K; p.NT = L.NT; p.G = L.G; p.group = L.group;
  p.KB = L.K / kstage;  // iterations (stages) per tile
  p.a_global = a_global;
  p.gated = L.gated;
  p.M = M;
  p.moe = moe;
  p.E = E;
  p.offsets = offsets;
  p.perm = perm;
  // FP8: per-token scales in the epilogue, caller row perm[r] / div for MoE;
  // the block scales were laid out per token tile above
  p.row_scale = L.bs == BS_F8 ? (const float *)a_scales : nullptr;
  p.a_div = a_div;
  p.gather = gather;
  p.out = (uint16_t *)out;
  p.ntw = t.ntw;
  p.mtiles = t.mtiles;
  p.nctas = t.nctas;
  // weights read by one token tile (dense), or by about one per expert (MoE):
  // stream them past L2 so that the activation tiles stay resident
  p.weights_once = ((!moe && t.mtiles == 1) || (moe && t.mtiles <= 2 * E)) ? 1 : 0;
  p.a_sf = (const uint8_t *)sf_tiles;
  p.a_sf_ld = 0;
  p.a_rows = a_rows;
  p.counters = (int *)workspace;
  p.partial = (float *)((uint8_t *)workspace + tc_counter_bytes(t));
  if (L.bs == BS_MX) return bs_launch_kind<BS_MX>(wm, am, p, t, st);
  if (L.bs == BS_F8) return bs_launch_kind<BS_F8>(wm, am, p, t, st);
  if (L.bs == BS_F8B) {
    switch (t.bnt) {
      case 16: return bsf_launch_one<16>(wm, am, p, t, st);
      case 32: return bsf_launch_one<32>(wm, am, p, t, st);
      case 64: return bsf_launch_one<64>(wm, am, p, t, st);
      case 128: return bsf_launch_one<128>(wm, am, p, t, st);
      default: return HQ_ERR_UNSUPPORTED;
    }
  }
  return bs_launch_kind<BS_NV>(wm, am, p, t, st);
}

}  // namespace hq
