// Tensor-core quantised-weight GEMM for few tokens per tile (16 or 32): the
// decode and small-batch regime, where the packed weight bytes set the time.
//
// "Announcing Humming", section "Tuning and JIT compilation per workload":
// for small batches the weight stream must saturate HBM, and the work is
// split along K so that every SM streams weights.  The sm_100a design:
//
//   * one persistent CTA per SM (736 threads, all of TMEM):
//       warps 0..3   epilogue: tcgen05.ld of the fp32 accumulator (warp w owns
//                    TMEM lanes 32w..32w+31), scales, bf16 out, or fp32
//                    partials and a per-warp last-arriver fixup;
//       warp 4       weight producer: one 1-D bulk copy each for the packed
//                    weights, the scales and the zero points of a stage;
//       warp 5       MMA issuer: tcgen05.mma with the dequantised weights as
//                    operand A in TMEM and the activations as operand B in
//                    shared memory, issued by one elected lane;
//       warps 6..21  dequant: NGRP groups of four warps (one per TMEM lane
//                    quadrant = 32 weight rows); group g decodes 64-k blocks
//                    g, g + NGRP, ... of every stage and stores each with one
//                    tcgen05.st.32x32b.x32;
//       warp 22      activation producer: one 3-D TMA per stage;
//   * a stage is four 64-k blocks (16 KB of 4-bit weights); the handshakes
//     (full / consumed / decoded / MMA done) are per stage, not per block;
//   * Stream-K: the (tile, k-block) iterations are cut into equal contiguous
//     ranges, one per CTA, so every SM streams the same number of weight
//     bytes; a tile shared by several CTAs is summed in k order by the last
//     CTA to finish its part (deterministic).
//   * every mbarrier wait is bounded (~1 s); on a timeout the CTA records
//     HQ_ERR_TIMEOUT, raises its abort flag, releases TMEM and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "hq_internal.cuh"

namespace hq {

namespace dec {

using tc::BM;
using tc::Traits;
using tc::Params;
using tc::TileInfo;

constexpr int NDQ = 16;                 // dequant warps (NGRP groups x 4 lane quadrants)
constexpr int NGRP = NDQ / 4;
constexpr int WARP_PRODUCER = 4, WARP_MMA = 5, WARP_DQ0 = 6;
constexpr int WARP_ACT = WARP_DQ0 + NDQ;  // activation producer
constexpr int THREADS = (WARP_ACT + 1) * 32;
constexpr int KPS = 4;                  // 64-k blocks per stage
constexpr int BPW = KPS / NGRP;         // blocks each dequant warp decodes per stage
static_assert(KPS % NGRP == 0, "stage blocks split evenly over the dequant groups");
constexpr int TMEM_COLS = 512;

template <int WF, int BNT, bool F8>
struct Cfg {
  static constexpr int A_COLS = F8 ? 16 : 32;          // TMEM columns per 64-k block
  static constexpr int ACT_KB = BNT * (F8 ? 64 : 128);  // one block of activations
  static constexpr int ACT = KPS * ACT_KB;              // [KPS][BNT][64], swizzled
  static constexpr int WPK = KPS * Traits<WF>::unit;
  static constexpr int SC = KPS * Traits<WF>::max_groups_kb * BM * Traits<WF>::sbytes;
  static constexpr int ZP = Traits<WF>::has_zero ? KPS * Traits<WF>::max_groups_kb * BM : 0;
  static constexpr int STAGE = (ACT + WPK + SC + ZP + 1023) / 1024 * 1024;
  static constexpr int NS_FIT = (200 * 1024) / STAGE;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;   // shared-memory ring depth
  static constexpr int CTRL = 8192;
  static constexpr int BYTES = NS * STAGE + CTRL + 1024;
  static constexpr int ND = 2;                          // accumulator buffers
  static constexpr int AS_COLS = KPS * A_COLS;          // TMEM columns per decoded stage
  static constexpr int NAS_FIT = (TMEM_COLS - ND * BNT) / AS_COLS;
  static constexpr int NAS = NAS_FIT > 4 ? 4 : NAS_FIT;  // TMEM A ring depth (stages)
  static constexpr int D_COL = NAS * AS_COLS;
  static_assert(NS >= 3, "stage too large");
  static_assert(NAS >= 2 && D_COL + ND * BNT <= TMEM_COLS, "TMEM budget");
};

// ---- Stream-K partition ------------------------------------------------------------
__device__ __forceinline__ long long range_begin(int c, long long total, int nctas) {
  return (long long)c * total / nctas;
}
// The CTA whose range holds iteration i.
__device__ __forceinline__ int cta_of(long long i, long long total, int nctas) {
  int c = (int)(((i + 1) * nctas - 1) / total);
  if (c >= nctas) c = nctas - 1;
  while (c + 1 < nctas && range_begin(c + 1, total, nctas) <= i) ++c;
  while (c > 0 && range_begin(c, total, nctas) > i) --c;
  return c;
}

// Walks a CTA's iterations in stages of up to KPS k-blocks that never cross
// a tile boundary.  Every role walks the same sequence.
struct Walk {
  int t, kb, left, n;
  bool seg_first, seg_last;
  __device__ __forceinline__ void start(long long beg, long long end, int KB) {
    t = (int)(beg / KB);
    kb = (int)(beg - (long long)t * KB);
    left = (int)(end - beg);
    seg_first = true;
    set(KB);
  }
  __device__ __forceinline__ void set(int KB) {
    n = min(KPS, min(KB - kb, left));
    seg_last = (kb + n == KB) || (n == left);
  }
  __device__ __forceinline__ void next(int KB) {
    left -= n;
    kb += n;
    seg_first = (kb == KB);
    if (kb == KB) {
      kb = 0;
      ++t;
    }
    set(KB);
  }
};

// Ring position: index and phase advanced together (no division).
struct Ring {
  int idx, phase;
  __device__ __forceinline__ void init() { idx = 0; phase = 0; }
  __device__ __forceinline__ void next(int n) {
    if (++idx == n) {
      idx = 0;
      phase ^= 1;
    }
  }
};

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y, int z, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// Decode one 64-k block of weight row r (packed layout: chunks of 16 bytes
// per row, [chunk][128 rows][16 B]) into bf16 pairs in k order.  `sc`/`zp`
// point at the stage's scales / zero points ([group - g0][128]).
template <int WF>
__device__ __forceinline__ void decode_bf16(const uint8_t *wpk, const uint8_t *sc, const uint8_t *zp, int r,
                                            int kbase, int g0, int gshift, uint32_t (&rg)[32]) {
  using TR = Traits<WF>;
  if constexpr (fmt_lowbit(WF)) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gt = ((kbase + 32 * h) >> gshift) - g0;
      uint32_t s2, z2;
      tc::lowbit_scale_zero<WF>(sc, zp, gt, r, s2, z2);
      tc::decode_half_lowbit<WF>(wpk, s2, z2, r, h, rg + 16 * h);
    }
  } else if constexpr (TR::wbits == 4) {
    uint32_t s2c = 0, z2c = 0;  // INT4 / UINT4: scale and zero point of the previous chunk
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const uint4 v = *reinterpret_cast<const uint4 *>(wpk + c * (BM * 16) + r * 16);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      const int gt = ((kbase + 32 * c) >> gshift) - g0;  // group of this chunk's first k
      if constexpr (WF == W_INT4 || WF == W_UINT4 || WF == W_MXINT4) {
        // groups are >= 32 k: one scale (and zero point) per chunk, loaded
        // again only when the second chunk starts a new group (MXINT4: the
        // E8M0 power of two as a bf16, exact)
        if (c == 0 || (gshift < 6 && gt != ((kbase >> gshift) - g0))) {
          s2c = WF == W_MXINT4 ? tc::bcast16(tc::e8m0_code_to_bf16(sc[gt * BM + r]))
                               : tc::bcast16(reinterpret_cast<const uint16_t *>(sc)[gt * BM + r]);
          // bf16 pair 128 + z in both halves, one multiply-add
          z2c = (WF == W_UINT4) ? 0x43004300u + (uint32_t)zp[gt * BM + r] * 0x10001u : 0x43084308u;
        }
        const uint32_t s2 = s2c, z2 = z2c;
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            rg[c * 16 + j * 4 + i] =
                tc::bmul2(tc::bsub2(((w4[j] >> (4 * i)) & 0x000F000Fu) | 0x43004300u, z2), s2);
      } else {
        // MXFP4: one group of 32 per chunk; NVFP4: two groups of 16 (words 0-1, 2-3)
        uint32_t s2[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const uint32_t code = sc[(gt + (WF == W_NVFP4 ? q : 0)) * BM + r];
          s2[q] = tc::bcast16(WF == W_MXFP4 ? tc::e8m0_code_to_bf16(code) : tc::e4m3_code_to_bf16(code));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            rg[c * 16 + j * 4 + i] = tc::bmul2(tc::bmul2(tc::e2m1_pair(w4[j] >> (4 * i)), 0x7E807E80u), s2[j >> 1]);
      }
    }
  } else {
    // 8-bit E4M3 weights with bf16 activations: four 16-k chunks
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = *reinterpret_cast<const uint4 *>(wpk + c * (BM * 16) + r * 16);
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        rg[c * 8 + j * 2] = tc::bmul2(tc::e4m3_pair(w4[j]), 0x7B807B80u);
        rg[c * 8 + j * 2 + 1] = tc::bmul2(tc::e4m3_pair(w4[j] >> 8), 0x7B807B80u);
      }
    }
  }
}

// One epilogue warp's end of a segment (Stream-K piece of a tile): v[m] is
// the fp32 accumulator of weight row n for the tile's token m.  A whole tile
// is scaled and written as bf16; a piece is stored as an fp32 partial
// (slot 0 for a head piece that starts mid-tile, else slot 1) and the warp
// takes its ticket for the tile: the last of the CTAs sharing the tile sums
// every part in k order and writes the rows.  `ki` = iterations per tile,
// `total` = iterations of the launch.
template <int BNT>
__device__ __forceinline__ void store_rows(const Params &p, const TileInfo &ti, int n, const float (&x)[BNT],
                                           float cs, float gs) {
  // output rows (and per-token scales) of the tile's tokens: one load per
  // lane, handed to the other lanes by shuffles (whole warp, BNT <= 32)
  const int lane = threadIdx.x & 31;
  int orow_l = 0;
  float rs_l = 1.f;
  if (lane < BNT && lane < ti.nvalid) {
    const int pos = ti.base + lane;
    orow_l = p.moe ? p.perm[pos] : pos;
    if (p.row_scale) rs_l = p.row_scale[p.moe ? orow_l / p.a_div : pos];
  }
  auto stores = [&](auto gated) {
#pragma unroll
    for (int m = 0; m < BNT; ++m) {
      const int orow = __shfl_sync(0xffffffffu, orow_l, m);
      const float rs = __shfl_sync(0xffffffffu, rs_l, m);
      float z = x[m];
      if (p.row_scale) z *= rs;
      z *= cs;
      z *= gs;
      tc::put_out<decltype(gated)::value>(p, orow, n, z, m < ti.nvalid && n < p.N);
    }
  };
  if (p.gated) stores(tc::GatedTag<true>{});
  else stores(tc::GatedTag<false>{});
}

template <int BNT>
__device__ __forceinline__ void finish_segment(const Params &p, const TileInfo &ti, int t, bool whole, bool head,
                                               const float (&v)[BNT], float cs, float gs, int cta, int warp,
                                               int lane, long long total, int ki) {
  const int r = warp * 32 + lane;
  const int n = ti.wt * BM + r;
  if (whole) {
    store_rows<BNT>(p, ti, n, v, cs, gs);
    return;
  }
  float *part = p.partial + ((size_t)cta * 2 + (head ? 0 : 1)) * BNT * BM;
#pragma unroll
  for (int m = 0; m < BNT; ++m) __stcg(&part[(size_t)m * BM + r], v[m]);
  __threadfence();
  __syncwarp();
  const long long t_first = (long long)t * ki;
  const int c_first = cta_of(t_first, total, p.nctas);
  const int c_last = cta_of(t_first + ki - 1, total, p.nctas);
  int last = 0;
  if (lane == 0) {
    int *ctr = p.counters + (size_t)t * 4 + warp;
    last = (atomicAdd(ctr, 1) == c_last - c_first);
    if (last) *ctr = 0;  // ready for the next call
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (!last) return;
  __threadfence();
  // contributors in k order; the loads of U contributors are in flight together
  constexpr int U = BNT <= 16 ? 2 : 1;  // within the 80-register budget of this kernel
  float x[BNT];
#pragma unroll
  for (int m = 0; m < BNT; ++m) x[m] = 0.f;
  for (int c0 = c_first; c0 <= c_last; c0 += U) {
    float y[U][BNT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u;
      if (c <= c_last) {
        const float *pc = p.partial + ((size_t)c * 2 + (c == c_first ? 1 : 0)) * BNT * BM + r;
#pragma unroll
        for (int m = 0; m < BNT; ++m) y[u][m] = __ldcg(pc + (size_t)m * BM);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (c0 + u <= c_last) {
#pragma unroll
        for (int m = 0; m < BNT; ++m) x[m] += y[u][m];
      }
  }
  store_rows<BNT>(p, ti, n, x, cs, gs);
}

template <int WF, int BNT, bool F8>
__global__ void __launch_bounds__(THREADS, 1) dec_gemm_kernel(const __grid_constant__ CUtensorMap act_map,
                                                               const Params p) {
  using TR = Traits<WF>;
  using C = Cfg<WF, BNT, F8>;
  static_assert(!F8 || WF == W_FP8, "the E4M3 x E4M3 path takes FP8 weights");
  constexpr int NS = C::NS, ND = C::ND, NAS = C::NAS;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle, by offsetting from the
  // shared array itself so that the compiler keeps every access an ld.shared
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t *ctrl = smem + NS * C::STAGE;
  uint64_t *full = reinterpret_cast<uint64_t *>(ctrl);  // [NS] stage landed
  uint64_t *sfree = full + NS;                           // [NS] stage consumed (MMA done)
  uint64_t *afull = sfree + NS;                          // [NAS] decoded stage in TMEM
  uint64_t *aempty = afull + NAS;                        // [NAS] decoded stage consumed by the MMA
  uint64_t *accf = aempty + NAS;                         // [ND] accumulator complete
  uint64_t *acce = accf + ND;                            // [ND] accumulator drained
  long long *s_total = reinterpret_cast<long long *>(acce + ND);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(s_total + 1);
  int *s_abort = reinterpret_cast<int *>(tmem_slot + 1);
  int *s_tpre = s_abort + 1;  // [E+1] MoE: prefix of token tiles per expert

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
      *s_total = (long long)tvalid * p.ntw * p.KB;  // (tile, k-block) iterations
      *s_abort = 0;
    }
  }
  if (tid == 32) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 2);  // weight and activation producers
      mbar_init(&sfree[s], 1);  // MMA commit: it runs after every dequant warp is done with the stage
    }
    for (int a = 0; a < NAS; ++a) {
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
  // broadcast from lane 0 so that the compiler treats everything derived as warp-uniform
  const long long total = __shfl_sync(0xffffffffu, *s_total, 0);
  const long long beg = range_begin(cta, total, p.nctas);
  const long long end = range_begin(cta + 1, total, p.nctas);
  if (beg >= end) return;

  // tile index -> weight tile, expert, token rows
  auto tile_info = [&](int t) {
    TileInfo ti;
    const int slot = t / p.ntw;
    ti.wt = t - slot * p.ntw;
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

  // The producer warps start loading at once; the warps that use tensor
  // memory wait (named barrier 1) for warp 0's allocation.
  const bool producer = (warp == WARP_PRODUCER || warp == WARP_ACT);
  uint32_t tmem = 0;
  if (producer) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(&act_map) : "memory");
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

  if (warp == WARP_PRODUCER) {
    // ================= weight producer (whole warp in step, lane 0 issues) =================
    // Packed weights, scales and zero points of each stage: three 1-D bulk
    // copies.  The activations come from their own producer warp, so that
    // the copy engine always has the next stage's requests queued.
    const uint64_t pol = p.weights_once ? policy_evict_first() : policy_evict_normal();
    Walk w;
    w.start(beg, end, p.KB);
    Ring rs;
    rs.init();
    int cur_t = -1;
    const uint8_t *wsrc = nullptr, *ssrc = nullptr, *zsrc = nullptr;  // current tile's streams
    for (int is = 0; w.left > 0; ++is, w.next(p.KB), rs.next(NS)) {
      if (w.t != cur_t) {
        const TileInfo ti = tile_info(w.t);
        const uint8_t *eb = p.packed + (size_t)ti.expert * p.stride;
        wsrc = eb + p.w_off + (size_t)ti.wt * p.KB * TR::unit;
        ssrc = eb + p.s_off + (size_t)ti.wt * p.G * BM * TR::sbytes;
        zsrc = eb + p.z_off + (size_t)ti.wt * p.G * BM;
        cur_t = w.t;
      }
      if (is >= NS && !mbar_wait(&sfree[rs.idx], rs.phase ^ 1)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      if (lane == 0) {
        uint8_t *st = smem + rs.idx * C::STAGE;
        const int g0 = (w.kb * TILE_K) >> p.gshift;
        const int g1 = (((w.kb + w.n) * TILE_K - 1) >> p.gshift) + 1;
        const uint32_t sb = TR::has_scales ? (uint32_t)((g1 - g0) * BM * TR::sbytes) : 0u;
        const uint32_t zb = TR::has_zero ? (uint32_t)((g1 - g0) * BM) : 0u;
        mbar_arrive_expect_tx(&full[rs.idx], TR::unit * w.n + sb + zb);
        bulk_g2s_stream(st + C::ACT, wsrc + (size_t)w.kb * TR::unit, TR::unit * w.n, &full[rs.idx], pol);
        if (TR::has_scales) bulk_g2s(st + C::ACT + C::WPK, ssrc + (size_t)g0 * BM * TR::sbytes, sb, &full[rs.idx]);
        if (TR::has_zero) bulk_g2s(st + C::ACT + C::WPK + C::SC, zsrc + (size_t)g0 * BM, zb, &full[rs.idx]);
      }
      __syncwarp();
    }
  } else if (warp == WARP_ACT) {
    // ================= activation producer: one 3-D TMA per stage, or =================
    // ================= (MoE indexed mode) 4-row gathers per 64-k block =================
    Walk w;
    w.start(beg, end, p.KB);
    Ring rs;
    rs.init();
    int cur_t = -1, base = 0, nvalid = 0, my_row = 0;
    for (int is = 0; w.left > 0; ++is, w.next(p.KB), rs.next(NS)) {
      if (w.t != cur_t) {
        const TileInfo ti = tile_info(w.t);
        base = ti.base;
        nvalid = ti.nvalid;
        cur_t = w.t;
        // indexed mode: lane i holds the caller row of the tile's row i
        // (rows past the valid ones repeat the last: loaded, never written back)
        if (p.gather) my_row = p.perm[base + min(lane, nvalid - 1)] / p.a_div;
      }
      if (is >= NS && !mbar_wait(&sfree[rs.idx], rs.phase ^ 1)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      uint8_t *st = smem + rs.idx * C::STAGE;
      if (!p.gather) {
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[rs.idx], (uint32_t)C::ACT);
          // box {64 k, BNT rows, KPS blocks}
          tma_load_3d(st, &act_map, 0, base, w.kb, &full[rs.idx]);
        }
      } else {
        const int ng = (nvalid + 3) >> 2;  // 4-row gathers per 64-k block
        if (lane == 0) mbar_arrive_expect_tx(&full[rs.idx], (uint32_t)(w.n * ng * 4 * 128));
        __syncwarp();
        // lane 4 * gi + j issues the gather of rows 4gi..4gi+3 for block j
        // (BNT <= 32: at most 8 groups x 4 blocks), all lanes at once
        const int gi = lane >> 2, j = lane & 3;
        const int r0 = __shfl_sync(0xffffffffu, my_row, (4 * gi) & 31);
        const int r1 = __shfl_sync(0xffffffffu, my_row, (4 * gi + 1) & 31);
        const int r2 = __shfl_sync(0xffffffffu, my_row, (4 * gi + 2) & 31);
        const int r3 = __shfl_sync(0xffffffffu, my_row, (4 * gi + 3) & 31);
        if (gi < ng && j < w.n)
          tc::tma_gather4(st + j * C::ACT_KB + gi * 512, &act_map, (w.kb + j) * TILE_K, r0, r1, r2, r3,
                          &full[rs.idx]);
      }
      __syncwarp();
    }
  } else if (warp >= WARP_DQ0 && warp < WARP_ACT) {
    // ================= dequant: warp = 32 weight rows of blocks grp, grp + NGRP, ... =================
    const int sp = warp & 3;                // TMEM lane quadrant this warp may access
    const int grp = (warp - WARP_DQ0) >> 2;  // first 64-k block of each stage (then every NGRP-th)
    const int r = sp * 32 + lane;           // weight row inside the tile
    const uint32_t t_row = tmem + ((uint32_t)(sp * 32) << 16);
    Walk w;
    w.start(beg, end, p.KB);
    Ring rs, ra;
    rs.init();
    ra.init();
    for (int is = 0; w.left > 0; ++is, w.next(p.KB), rs.next(NS), ra.next(NAS)) {
      if (!mbar_wait(&full[rs.idx], rs.phase)) { *s_abort = 1; break; }
      if (is >= NAS && !mbar_wait(&aempty[ra.idx], ra.phase ^ 1)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      tc::tc_fence_after();
#pragma unroll
      for (int b = 0; b < BPW; ++b) {
        const int blk = grp + b * NGRP;  // 64-k block of the stage
        if (blk < w.n) {
          const uint8_t *st = smem + rs.idx * C::STAGE;
          const uint8_t *wpk = st + C::ACT + blk * TR::unit;
          const uint32_t taddr = t_row + (uint32_t)(ra.idx * C::AS_COLS + blk * C::A_COLS);
          if constexpr (F8) {
            // E4M3 weights go to TMEM unchanged, bytes put back in k order
            uint32_t rg8[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 v = *reinterpret_cast<const uint4 *>(wpk + c * (BM * 16) + r * 16);
              rg8[c * 4 + 0] = __byte_perm(v.x, 0, 0x3120);
              rg8[c * 4 + 1] = __byte_perm(v.y, 0, 0x3120);
              rg8[c * 4 + 2] = __byte_perm(v.z, 0, 0x3120);
              rg8[c * 4 + 3] = __byte_perm(v.w, 0, 0x3120);
            }
            tc::tmem_st16(taddr, rg8);
          } else {
            const int g0 = (w.kb * TILE_K) >> p.gshift;
            uint32_t rg[32];
            decode_bf16<WF>(wpk, st + C::ACT + C::WPK, st + C::ACT + C::WPK + C::SC, r, (w.kb + blk) * TILE_K, g0,
                            p.gshift, rg);
            tmem_st32(taddr, rg);
          }
        }
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&afull[ra.idx]);
    }
  } else if (warp == WARP_MMA) {
    // ================= MMA issuer (whole warp in step, one elected lane issues) =================
    constexpr uint32_t idesc = F8 ? tc::idesc_e4m3<BNT>() : tc::idesc_bf16<BNT>();
    Walk w;
    w.start(beg, end, p.KB);
    Ring rs, ra, rd;
    rs.init();
    ra.init();
    rd.init();
    int q = 0;  // segments started
    for (int is = 0; w.left > 0; ++is, w.next(p.KB), rs.next(NS), ra.next(NAS)) {
      if (w.seg_first) {
        if (q > 0) rd.next(ND);
        if (q >= ND && !mbar_wait(&acce[rd.idx], rd.phase ^ 1)) { *s_abort = 1; break; }
        ++q;
      }
      if (!mbar_wait(&full[rs.idx], rs.phase)) { *s_abort = 1; break; }
      if (!mbar_wait(&afull[ra.idx], ra.phase)) { *s_abort = 1; break; }
      if (*(volatile int *)s_abort) break;
      tc::tc_fence_after();
      // operands are warp-uniform (they live in uniform registers); one
      // elected lane issues the stage's MMAs back to back
      const uint32_t tmem_d = tmem + (uint32_t)(C::D_COL + rd.idx * BNT);
      const uint32_t a_col = tmem + (uint32_t)(ra.idx * C::AS_COLS);
      const uint32_t b_addr = smem_u32(smem + rs.idx * C::STAGE);
      const uint64_t bdesc0 = F8 ? tc::sw64_desc(b_addr) : tc::sw128_desc(b_addr);
      const uint32_t acc0 = w.seg_first ? 0u : 1u;
      if (elect_one()) {
#pragma unroll
        for (int j = 0; j < KPS; ++j) {
          if (j < w.n) {
            const uint64_t bdesc = bdesc0 + (uint64_t)((j * C::ACT_KB) >> 4);
            if constexpr (F8) {
#pragma unroll
              for (int k32 = 0; k32 < 2; ++k32)
                tc::mma_ts_f8(tmem_d, a_col + (uint32_t)(j * C::A_COLS + k32 * 8), bdesc + (uint64_t)(k32 * 2), idesc,
                              (j > 0 || k32 > 0) ? 1u : acc0);
            } else {
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16)
                tc::mma_ts(tmem_d, a_col + (uint32_t)(j * C::A_COLS + k16 * 8), bdesc + (uint64_t)(k16 * 2), idesc,
                           (j > 0 || k16 > 0) ? 1u : acc0);
            }
          }
        }
        tc::mma_commit(&aempty[ra.idx]);
        tc::mma_commit(&sfree[rs.idx]);
        if (w.seg_last) tc::mma_commit(&accf[rd.idx]);
      }
      __syncwarp();
    }
  } else {
    // ================= epilogue: warps 0..3, thread = weight row =================
    const int r = warp * 32 + lane;
    Ring rd;
    rd.init();
    int t = (int)(beg / p.KB);
    int kb0 = (int)(beg - (long long)t * p.KB);
    int left = (int)(end - beg);
    for (int q = 0; left > 0; ++q, rd.next(ND)) {
      const int seg_len = min(p.KB - kb0, left);
      const bool whole = (kb0 == 0) && (seg_len == p.KB);
      const bool ok = mbar_wait(&accf[rd.idx], rd.phase);
      tc::tc_fence_after();
      if (!ok || *(volatile int *)s_abort) break;
      const TileInfo ti = tile_info(t);
      const uint8_t *eb = p.packed + (size_t)ti.expert * p.stride;
      const int n = ti.wt * BM + r;
      float cs = 1.f, gs = 1.f;
      if (WF == W_FP8 && n < p.N) cs = reinterpret_cast<const float *>(eb + p.c_off)[n];
      if (WF == W_NVFP4) gs = reinterpret_cast<const float *>(eb + p.g_off)[0];
      if (p.a_global) gs = __fmul_rn(gs, *p.a_global);
      float v[BNT];
#pragma unroll
      for (int c0 = 0; c0 < BNT; c0 += 16) {
        float v16[16];
        tc::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(C::D_COL + rd.idx * BNT + c0), v16);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[c0 + i] = v16[i];
      }
      // accumulator read: hand it back to the MMA warp
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[rd.idx]);
      finish_segment<BNT>(p, ti, t, whole, kb0 > 0, v, cs, gs, cta, warp, lane, total, p.KB);
      left -= seg_len;
      ++t;
      kb0 = 0;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

}  // namespace dec

// ---- host side -------------------------------------------------------------------

// [rows, K] row-major activations viewed as {64 k, rows, K/64 blocks}; box =
// {64, box_rows, 4}: bf16 with a 128-byte swizzle or E4M3 bytes with a 64-byte
// swizzle, landing in shared memory as [4 blocks][box_rows][64].
bool make_act_map_3d(CUtensorMap *m, const void *a, int rows, int K, int box_rows, bool e4m3) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int es = e4m3 ? 1 : 2;
  cuuint64_t dims[3] = {64u, (cuuint64_t)rows, (cuuint64_t)(K / 64)};
  cuuint64_t strides[2] = {(cuuint64_t)K * es, (cuuint64_t)64 * es};
  cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, (cuuint32_t)dec::KPS};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void *>(a), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        e4m3 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int WF, int BNT, bool F8>
static hq_status dec_launch_one(const CUtensorMap &map, const tc::Params &p, const TcLaunch &t, cudaStream_t st) {
  using C = dec::Cfg<WF, BNT, F8>;
  auto kern = dec::dec_gemm_kernel<WF, BNT, F8>;
  static unsigned configured = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
  if (dev >= 32 || !(configured & (1u << dev))) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES) != cudaSuccess)
      return HQ_ERR_CUDA;
    if (dev < 32) configured |= 1u << dev;
  }
  kern<<<t.nctas, dec::THREADS, C::BYTES, st>>>(map, p);
  return check_launch();
}

template <int WF, bool F8 = false>
static hq_status dec_launch_wf(const CUtensorMap &map, const tc::Params &p, const TcLaunch &t, cudaStream_t st) {
  if (t.bnt == 16) return dec_launch_one<WF, 16, F8>(map, p, t, st);
  return dec_launch_one<WF, 32, F8>(map, p, t, st);
}

hq_status launch_dec_gemm(const Layout &L, const tc::Params &p, const void *a, int a_rows, const TcLaunch &t,
                          cudaStream_t st, bool e4m3_act) {
  CUtensorMap map;
  // indexed mode: a 2-D map of the caller's rows with one-row boxes for the
  // 4-row gathers (bf16 only); otherwise the 3-D map of KPS blocks per box
  if (p.gather ? !make_act_map(&map, a, a_rows, L.K, 1, false)
               : !make_act_map_3d(&map, a, a_rows, L.K, t.bnt, e4m3_act))
    return HQ_ERR_CUDA;
  switch (L.fmt) {
    case W_INT4: return dec_launch_wf<W_INT4>(map, p, t, st);
    case W_E0M3: return dec_launch_wf<W_INT4>(map, p, t, st);  // packed as INT4
    case W_MXINT4: return dec_launch_wf<W_MXINT4>(map, p, t, st);
    case W_INT1: return dec_launch_wf<W_INT1>(map, p, t, st);
    case W_UINT1: return dec_launch_wf<W_UINT1>(map, p, t, st);
    case W_INT2: return dec_launch_wf<W_INT2>(map, p, t, st);
    case W_UINT2: return dec_launch_wf<W_UINT2>(map, p, t, st);
    case W_INT3: return dec_launch_wf<W_INT3>(map, p, t, st);
    case W_UINT3: return dec_launch_wf<W_UINT3>(map, p, t, st);
    case W_E2M3: return dec_launch_wf<W_E2M3>(map, p, t, st);
    case W_E3M2: return dec_launch_wf<W_E3M2>(map, p, t, st);
    case W_UINT4: return dec_launch_wf<W_UINT4>(map, p, t, st);
    case W_MXFP4: return dec_launch_wf<W_MXFP4>(map, p, t, st);
    case W_NVFP4: return dec_launch_wf<W_NVFP4>(map, p, t, st);
    case W_FP8: return e4m3_act ? dec_launch_wf<W_FP8, true>(map, p, t, st) : dec_launch_wf<W_FP8>(map, p, t, st);
    default: return HQ_ERR_UNSUPPORTED;
  }
}

}  // namespace hq
