// C-ABI entry points of libhq: argument validation, workspace planning and
// kernel dispatch.  Every call validates on the host, launches on the
// caller's stream, allocates nothing and never synchronises (except
// hq_device_error, whose job is to synchronise).
#include <cuda_runtime.h>

#include <cstring>

#include "hq_internal.cuh"

namespace hq {

hq_status launch_pack(const Layout &L, int E, const void *codes, const void *scales, const void *zeros,
                      const float *global_scale, void *packed, cudaStream_t st);
hq_status launch_unpack(const Layout &L, int E, const void *packed, void *codes, void *scales, void *zeros,
                        float *global_scale, cudaStream_t st);
hq_status launch_quant_act(int afmt, int M, int K, const void *x, void *codes, void *scales, float *global_out,
                           const float *static_global, void *workspace, cudaStream_t st);
hq_status launch_act_decode(int afmt, int R, int K, const void *codes, const void *scales, const int32_t *idx,
                            int div, void *out, cudaStream_t st);
hq_status launch_gather_rows(int R, int K, const void *a, const int32_t *idx, int div, void *out, cudaStream_t st);
hq_status launch_moe_permute(int T, int topk, int E, const int32_t *ids, int32_t *offsets, int32_t *perm,
                             int32_t *inv, cudaStream_t st);
hq_status launch_unpermute_sum(int T, int topk, int N, const void *y, const int32_t *inv, const float *w, float rs,
                               void *out, cudaStream_t st);

hq_status launch_tc_gemm(const Layout &L, const void *packed, const void *a_bf16, int a_rows, const float *row_scale,
                         const float *a_global, int M, int moe, int E, const int32_t *offsets, const int32_t *perm,
                         int a_div, int gather, void *out, const TcLaunch &t, void *workspace, cudaStream_t st,
                         bool e4m3_act = false);

hq_status launch_bs_gemm(const Layout &L, const void *packed, int E, const void *a_codes, int a_rows,
                         const void *a_scales, int a_div, const float *a_global, int M, int moe,
                         const int32_t *offsets, const int32_t *perm, void *out, const TcLaunch &t,
                         void *workspace, void *sf_tiles, cudaStream_t st, int gather = 0);
size_t bs_sf_tiles_bytes(const Layout &L, const TcLaunch &t);
hq_status launch_gather_bytes(int R, int row_bytes, const void *a, const int32_t *idx, int div, void *out,
                              cudaStream_t st);
hq_status launch_quant_act_masked(int afmt, int E, int slab, int K, const void *x, const int32_t *counts,
                                  void *codes, void *scales, float *global_out, void *workspace, cudaStream_t st);
hq_status launch_moe_masked_prepare(int E, int slab, const int32_t *counts, int32_t *offsets, int32_t *perm,
                                    cudaStream_t st);
hq_status launch_silu_and_mul(int R, int I, const void *y, void *out, cudaStream_t st);

hq_status check_launch() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? HQ_OK : HQ_ERR_CUDA;
}

bool device_is_sm100() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return false;
  return major == 10 && minor == 0;
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Bytes of one activation row in its quantised storage and of its scales.
static size_t act_code_bytes(int afmt, int K) { return afmt == A_NVFP4 ? (size_t)K / 2 : (size_t)K; }
static size_t act_scale_bytes(int afmt, int K) {
  switch (afmt) {
    case A_FP8: return 4;
    case A_FP8G: return (size_t)K / 128 * 4;
    case A_MXFP8: return (size_t)K / 32;
    case A_NVFP4: return (size_t)K / 16;
    default: return 0;
  }
}

// ---- workspace carving: regions placed in order, 256-byte aligned --------
struct Carver {
  uint8_t *base;
  size_t off = 0;
  void *take(size_t bytes) {
    void *p = base ? base + off : nullptr;
    off = align_up(off + bytes, 256);
    return p;
  }
};

// Dense GEMM plan (shared by the size query and the call).
struct DensePlan {
  Layout L;
  int afmt;
  TcLaunch s;
};

static hq_status plan_dense(const hq_quant_desc *d, int M, int N, int K, DensePlan *pl) {
  int fmt, afmt;
  if (!d) return HQ_ERR_INVALID_ARG;
  if (!weight_format(d, &fmt) || !act_format(d, &afmt)) return HQ_ERR_UNSUPPORTED;
  if (M < 0 || N < 1 || !valid_k(d, K)) return HQ_ERR_INVALID_ARG;
  pl->L = layout_for(d, fmt, N, K);
  pl->afmt = afmt;
  if (!pair_supported(pl->L, afmt)) return HQ_ERR_UNSUPPORTED;
  pl->s = plan_tc(M > 0 ? M : 1, 0, N, pl->L.KB, false, pl->L.bs);
  return HQ_OK;
}

static int device_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    n = 148;
  return n > 0 ? n : 148;
}

// Dense plan with compute options.  Batch invariance: 64-token tiles and no
// K split, so that each output row is one tile's k-ordered sum whatever M:
// the multi-stage kernel with at most as many CTAs as tiles (whole tiles
// round-robin), or the TMA-fed kernel with a CTA count that divides the tile
// count (its contiguous per-CTA ranges then hold whole tiles).
static hq_status plan_dense_cfg(const hq_quant_desc *d, const hq_compute_config *cfg, int M, int N, int K,
                                DensePlan *pl) {
  const hq_status ps = plan_dense(d, M, N, K, pl);
  if (ps != HQ_OK || !cfg || !cfg->batch_invariant) return ps;
  for (int i = 0; i < 7; ++i)
    if (cfg->reserved[i] != 0) return HQ_ERR_INVALID_ARG;
  TcLaunch t{};
  t.bnt = 64;
  t.ntw = pl->L.NT;
  t.mtiles = M > 0 ? (M + 63) / 64 : 1;
  const long tiles = (long)t.ntw * t.mtiles;
  const int sms = device_sm_count();
  if (pl->L.bs == BS_NONE) {
    t.kind = 0;
    t.nctas = (int)(tiles < 2L * sms ? tiles : 2L * sms);  // two 64-token CTAs per SM
  } else {
    t.kind = 2;
    int n = (int)(tiles < sms ? tiles : sms);
    while (n > 1 && tiles % n != 0) --n;
    t.nctas = n;
  }
  pl->s = t;
  return HQ_OK;
}

// Pointer checks of a dense call (shared by every dense entry point, before
// anything is enqueued).
static hq_status dense_args(const DensePlan &pl, const void *packed_w, const void *a, const void *a_scales,
                            const float *a_global, const void *c_bf16) {
  if (!packed_w || !a || !c_bf16 || !aligned16(packed_w) || !aligned16(a)) return HQ_ERR_INVALID_ARG;
  if (pl.afmt != A_BF16 && !a_scales) return HQ_ERR_INVALID_ARG;
  if (pl.afmt == A_NVFP4 && !a_global) return HQ_ERR_INVALID_ARG;
  if (pl.L.bs != BS_NONE && ((uintptr_t)a_scales & 3u)) return HQ_ERR_INVALID_ARG;
  return HQ_OK;
}

// Dense workspace: split-K state; then either the decoded bf16 copy of
// quantised activations, or (block-scaled MMA) the activation scales in the
// kernel's chunk order.
static size_t dense_ws(const DensePlan &pl, int M, int K, uint8_t *base, void **split_ws, void **a_dec) {
  Carver c{base};
  *split_ws = c.take(tc_workspace_bytes(pl.s));
  if (pl.L.bs != BS_NONE) *a_dec = c.take(bs_sf_tiles_bytes(pl.L, pl.s));
  else *a_dec = (pl.afmt != A_BF16) ? c.take((size_t)M * K * 2) : nullptr;
  return c.off;
}

// MoE plan.
struct MoePlan {
  Layout L;
  int afmt;
  TcLaunch s;
  int R;         // routed rows = T * topk
  int src_rows;  // activation rows supplied by the caller
};

static hq_status plan_moe(const hq_quant_desc *d, int T, int topk, int E, int N, int K, int a_per_slot,
                          MoePlan *pl) {
  int fmt, afmt;
  if (!d) return HQ_ERR_INVALID_ARG;
  if (!weight_format(d, &fmt) || !act_format(d, &afmt)) return HQ_ERR_UNSUPPORTED;
  if (T < 0 || topk < 1 || E < 1 || E > 1024 || N < 1 || !valid_k(d, K)) return HQ_ERR_INVALID_ARG;
  if ((long)T * topk > (1L << 30)) return HQ_ERR_INVALID_ARG;
  pl->L = layout_for(d, fmt, N, K);
  pl->afmt = afmt;
  if (!pair_supported(pl->L, afmt)) return HQ_ERR_UNSUPPORTED;
  pl->R = T * topk;
  pl->src_rows = a_per_slot ? pl->R : T;
  const int R = pl->R > 0 ? pl->R : 1;
  const int active = R < E ? R : E;
  const int avg = (R + active - 1) / active;
  const int bnt = plan_tc(avg, 1, N, pl->L.KB, true, pl->L.bs).bnt;
  long bound = (R + bnt - 1) / bnt + active;
  if (bound > R) bound = R;
  pl->s = plan_tc(avg, (int)bound, N, pl->L.KB, true, pl->L.bs);
  return HQ_OK;
}

// Masked layout plan: E slabs of `slab` rows, of which expected_m are
// typically valid (the token tile follows it); R = E * slab rows bound the
// staging and the token tiles (at most ceil(slab / tile) per expert).
static hq_status plan_moe_masked(const hq_quant_desc *d, int E, int slab, int N, int K, int expected_m,
                                 MoePlan *pl) {
  int fmt, afmt;
  if (!d) return HQ_ERR_INVALID_ARG;
  if (!weight_format(d, &fmt) || !act_format(d, &afmt)) return HQ_ERR_UNSUPPORTED;
  if (E < 1 || E > 1024 || slab < 1 || N < 1 || !valid_k(d, K)) return HQ_ERR_INVALID_ARG;
  if ((long)E * slab > (1L << 30)) return HQ_ERR_INVALID_ARG;
  pl->L = layout_for(d, fmt, N, K);
  pl->afmt = afmt;
  if (!pair_supported(pl->L, afmt)) return HQ_ERR_UNSUPPORTED;
  pl->R = E * slab;
  pl->src_rows = E * slab;
  const int em = expected_m < 1 ? slab : (expected_m > slab ? slab : expected_m);
  const int bnt = plan_tc(em, 1, N, pl->L.KB, true, pl->L.bs).bnt;
  long bound = (long)E * ((slab + bnt - 1) / bnt);
  if (bound > pl->R) bound = pl->R;
  pl->s = plan_tc(em, (int)bound, N, pl->L.KB, true, pl->L.bs);
  return HQ_OK;
}

struct MoeWs {
  void *split, *y, *a_bf16, *codes, *scales, *glob, *amax;
  void *s_codes, *s_scales;  // block-scaled layouts: expert-sorted codes, scale chunks per token tile
  int32_t *r_off, *r_perm, *r_inv;  // routing prepared by the call itself (from topk_ids)
};

// Workspace of an MoE call.  Grouped mode stages the R routed rows
// expert-contiguous (bf16 rows for the dequantisation kernels, quantised
// codes for the block-scaled MMA); indexed mode stages nothing for bf16
// activations and only the caller's rows decoded to bf16 for quantised ones
// on the dequantisation path (src_rows rows, not R).  `route` adds room for
// the routing prepare of a call given topk_ids alone.
static size_t moe_ws(const MoePlan &pl, hq_moe_mode mode, int E, int K, int N, int combine, bool route,
                     uint8_t *base, MoeWs *w) {
  Carver c{base};
  const bool indexed = (mode == HQ_MOE_INDEXED);
  w->split = c.take(tc_workspace_bytes(pl.s));
  w->y = combine ? c.take((size_t)pl.R * N * 2) : nullptr;
  w->a_bf16 = w->s_codes = w->s_scales = nullptr;
  if (pl.L.bs == BS_NONE) {
    if (!indexed) w->a_bf16 = c.take((size_t)pl.R * K * 2);
    else if (pl.afmt != A_BF16) w->a_bf16 = c.take((size_t)pl.src_rows * K * 2);
  } else {
    if (!indexed) w->s_codes = c.take((size_t)pl.R * act_code_bytes(pl.afmt, K));
    w->s_scales = c.take(bs_sf_tiles_bytes(pl.L, pl.s));  // scales in the kernel's chunk order
  }
  if (pl.afmt != A_BF16) {
    w->codes = c.take((size_t)pl.src_rows * act_code_bytes(pl.afmt, K));
    w->scales = c.take((size_t)pl.src_rows * act_scale_bytes(pl.afmt, K));
    w->glob = c.take(16);
    w->amax = c.take(16);
  } else {
    w->codes = w->scales = w->glob = w->amax = nullptr;
  }
  w->r_off = w->r_perm = w->r_inv = nullptr;
  if (route) {
    w->r_off = (int32_t *)c.take((size_t)(E + 1) * sizeof(int32_t));
    w->r_perm = (int32_t *)c.take((size_t)pl.R * sizeof(int32_t));
    w->r_inv = (int32_t *)c.take((size_t)pl.R * sizeof(int32_t));
  }
  return c.off;
}

// The GEMM part of every MoE mode, given the routing (offsets, perm).
// Activation rows: bf16 `a`, quantised here when the description asks
// (`counts` selects the masked layout's quantiser), or the caller's codes
// (`a_scales` non-null).  Grouped mode copies the routed rows
// expert-contiguous first; indexed mode lets the GEMM gather the caller's
// rows through the routing index.  Then the optional weighted combine.
static hq_status moe_run(const MoePlan &pl, hq_moe_mode mode, int T, int topk, int E, int N, int K,
                         const void *packed_w, const void *a, const void *a_scales, const float *a_global, int div,
                         const int32_t *counts, const int32_t *expert_offsets, const int32_t *perm,
                         const float *topk_weights, float routed_scale, int combine, void *out_bf16, const MoeWs &w,
                         cudaStream_t st) {
  const bool indexed = (mode == HQ_MOE_INDEXED);
  hq_status s = HQ_OK;
  void *y = combine ? w.y : out_bf16;
  // quantised activation rows (src_rows of them): the caller's or our own
  const void *codes = a;
  const void *scales = a_scales;
  const float *glob = a_global;
  if (pl.afmt != A_BF16 && !a_scales) {
    s = counts ? launch_quant_act_masked(pl.afmt, E, pl.src_rows / E, K, a, counts, w.codes, w.scales,
                                         (float *)w.glob, w.amax, st)
               : launch_quant_act(pl.afmt, pl.src_rows, K, a, w.codes, w.scales, (float *)w.glob, nullptr, w.amax,
                                  st);
    if (s != HQ_OK) return s;
    codes = w.codes;
    scales = w.scales;
    glob = (const float *)w.glob;
  }
  if (pl.L.bs != BS_NONE) {
    // block-scaled MMA: the quantised codes go to the tensor core as they are
    const void *rows = codes;
    int a_rows = pl.src_rows;
    if (!indexed) {
      s = launch_gather_bytes(pl.R, (int)act_code_bytes(pl.afmt, K), codes, perm, div, w.s_codes, st);
      if (s != HQ_OK) return s;
      rows = w.s_codes;
      a_rows = pl.R;
    }
    s = launch_bs_gemm(pl.L, packed_w, E, rows, a_rows, scales, div, pl.afmt == A_NVFP4 ? glob : nullptr, 0, 1,
                       expert_offsets, perm, y, pl.s, w.split, w.s_scales, st, indexed ? 1 : 0);
  } else {
    const void *a_use = a;
    int a_rows = pl.src_rows;
    const float *row_scale = nullptr;
    const float *a_glob = nullptr;
    if (pl.afmt != A_BF16) {
      // decoded exactly to bf16: the caller's rows (indexed) or the routed rows (grouped)
      s = indexed ? launch_act_decode(pl.afmt, pl.src_rows, K, codes, scales, nullptr, 1, w.a_bf16, st)
                  : launch_act_decode(pl.afmt, pl.R, K, codes, scales, perm, div, w.a_bf16, st);
      if (s != HQ_OK) return s;
      a_use = w.a_bf16;
      a_rows = indexed ? pl.src_rows : pl.R;
      if (pl.afmt == A_FP8) row_scale = (const float *)scales;
      if (pl.afmt == A_NVFP4) a_glob = glob;
    } else if (!indexed) {
      s = launch_gather_rows(pl.R, K, a, perm, div, w.a_bf16, st);
      if (s != HQ_OK) return s;
      a_use = w.a_bf16;
      a_rows = pl.R;
    }
    s = launch_tc_gemm(pl.L, packed_w, a_use, a_rows, row_scale, a_glob, 0, 1, E, expert_offsets, perm, div,
                       indexed ? 1 : 0, y, pl.s, w.split, st);
  }
  if (s != HQ_OK) return s;
  if (combine) s = launch_unpermute_sum(T, topk, N, y, nullptr, topk_weights, routed_scale, out_bf16, st);
  return s;
}

}  // namespace hq

using namespace hq;

extern "C" {

const char *hq_status_string(hq_status s) {
  switch (s) {
    case HQ_OK: return "ok";
    case HQ_ERR_INVALID_ARG: return "invalid argument";
    case HQ_ERR_UNSUPPORTED: return "unsupported format combination or size";
    case HQ_ERR_WORKSPACE: return "workspace too small";
    case HQ_ERR_CUDA: return "CUDA error";
    case HQ_ERR_TIMEOUT: return "device-side wait timed out";
    case HQ_ERR_DEVICE_INDEX: return "expert id out of range";
    case HQ_ERR_ARCH: return "device is not sm_100";
    default: return "unknown status";
  }
}

// Self-test of the device-side failure path: one warp waits on an mbarrier
// that nothing arrives on, with the bounded wait every pipeline uses; the
// wait gives up after limit_ns, records HQ_ERR_TIMEOUT and the kernel returns.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, limit_ns);  // nothing arrives
}

hq_status hq_selftest_wait_timeout(unsigned long long limit_ns, hq_stream_t stream) {
  if (limit_ns == 0 || limit_ns > WAIT_LIMIT_NS) return HQ_ERR_INVALID_ARG;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns);
  return check_launch();
}

hq_status hq_device_error(hq_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return HQ_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_hq_error, sizeof(int)) != cudaSuccess) return HQ_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_hq_error, &zero, sizeof(int)) != cudaSuccess) return HQ_ERR_CUDA;
  return (hq_status)v;
}

size_t hq_packed_weights_bytes(const hq_quant_desc *desc, int E, int N, int K) {
  int fmt, afmt;
  if (!weight_format(desc, &fmt) || E < 1 || N < 1 || !valid_k(desc, K)) return 0;
  const Layout L = layout_for(desc, fmt, N, K);
  if (!act_format(desc, &afmt) || !pair_supported(L, afmt)) return 0;
  return L.stride * (size_t)E;
}

// Pack / unpack with the plain or the gated (gate/up rows side by side) row order.
static hq_status pack_impl(const hq_quant_desc *desc, int E, int N, int K, const void *codes, const void *scales,
                           const void *zeros, const float *global_scale, void *packed, hq_stream_t stream,
                           bool gated) {
  int fmt;
  if (!desc) return HQ_ERR_INVALID_ARG;
  if (!weight_format(desc, &fmt)) return HQ_ERR_UNSUPPORTED;
  if (E < 1 || N < 1 || !valid_k(desc, K)) return HQ_ERR_INVALID_ARG;
  if (gated && (N % TILE_N) != 0) return HQ_ERR_INVALID_ARG;
  if (!codes || !scales || !packed) return HQ_ERR_INVALID_ARG;
  if (fmt_zero(fmt) != (zeros != nullptr)) return HQ_ERR_INVALID_ARG;
  if ((fmt == W_NVFP4) != (global_scale != nullptr)) return HQ_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(packed) || ((uintptr_t)scales & 3u)) return HQ_ERR_INVALID_ARG;
  Layout L = layout_for(desc, fmt, N, K);
  int afmt;
  if (!act_format(desc, &afmt) || !pair_supported(L, afmt)) return HQ_ERR_UNSUPPORTED;
  if (gated && L.bs == BS_F8B) return HQ_ERR_UNSUPPORTED;  // a tile would span two scale blocks
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  L.gated = gated ? 1 : 0;
  return launch_pack(L, E, codes, scales, zeros, global_scale, packed, (cudaStream_t)stream);
}

static hq_status unpack_impl(const hq_quant_desc *desc, int E, int N, int K, const void *packed, void *codes,
                             void *scales, void *zeros, float *global_scale, hq_stream_t stream, bool gated) {
  int fmt;
  if (!desc) return HQ_ERR_INVALID_ARG;
  if (!weight_format(desc, &fmt)) return HQ_ERR_UNSUPPORTED;
  if (E < 1 || N < 1 || !valid_k(desc, K)) return HQ_ERR_INVALID_ARG;
  if (gated && (N % TILE_N) != 0) return HQ_ERR_INVALID_ARG;
  if (!codes || !scales || !packed) return HQ_ERR_INVALID_ARG;
  if (fmt_zero(fmt) != (zeros != nullptr)) return HQ_ERR_INVALID_ARG;
  if ((fmt == W_NVFP4) != (global_scale != nullptr)) return HQ_ERR_INVALID_ARG;
  Layout L = layout_for(desc, fmt, N, K);
  int afmt;
  if (!act_format(desc, &afmt) || !pair_supported(L, afmt)) return HQ_ERR_UNSUPPORTED;
  if (gated && L.bs == BS_F8B) return HQ_ERR_UNSUPPORTED;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  L.gated = gated ? 1 : 0;
  return launch_unpack(L, E, packed, codes, scales, zeros, global_scale, (cudaStream_t)stream);
}

hq_status hq_pack_weights(const hq_quant_desc *desc, int E, int N, int K, const void *codes, const void *scales,
                          const void *zeros, const float *global_scale, void *packed, hq_stream_t stream) {
  return pack_impl(desc, E, N, K, codes, scales, zeros, global_scale, packed, stream, false);
}

hq_status hq_unpack_weights(const hq_quant_desc *desc, int E, int N, int K, const void *packed, void *codes,
                            void *scales, void *zeros, float *global_scale, hq_stream_t stream) {
  return unpack_impl(desc, E, N, K, packed, codes, scales, zeros, global_scale, stream, false);
}

hq_status hq_pack_weights_gated(const hq_quant_desc *desc, int E, int N2, int K, const void *codes,
                                const void *scales, const void *zeros, const float *global_scale, void *packed,
                                hq_stream_t stream) {
  return pack_impl(desc, E, N2, K, codes, scales, zeros, global_scale, packed, stream, true);
}

hq_status hq_unpack_weights_gated(const hq_quant_desc *desc, int E, int N2, int K, const void *packed, void *codes,
                                  void *scales, void *zeros, float *global_scale, hq_stream_t stream) {
  return unpack_impl(desc, E, N2, K, packed, codes, scales, zeros, global_scale, stream, true);
}

hq_status hq_quant_act(const hq_quant_desc *desc, int M, int K, const void *x_bf16, void *codes, void *scales,
                       float *global_out, const float *static_global, void *workspace, size_t ws_bytes,
                       hq_stream_t stream) {
  int afmt;
  if (!desc) return HQ_ERR_INVALID_ARG;
  if (!act_format(desc, &afmt)) return HQ_ERR_UNSUPPORTED;
  if (afmt == A_BF16) return HQ_ERR_INVALID_ARG;
  if (M < 0 || K < 32 || (K % 32) != 0) return HQ_ERR_INVALID_ARG;
  if (afmt == A_FP8G && (K % 128) != 0) return HQ_ERR_INVALID_ARG;
  if (M == 0) return HQ_OK;
  if (!x_bf16 || !codes || !scales || !aligned16(x_bf16) || !aligned16(codes)) return HQ_ERR_INVALID_ARG;
  if (afmt == A_NVFP4) {
    if (!global_out && !static_global) return HQ_ERR_INVALID_ARG;
    if (!static_global && (!workspace || ws_bytes < 16)) return HQ_ERR_WORKSPACE;
  }
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  return launch_quant_act(afmt, M, K, x_bf16, codes, scales, global_out, static_global, workspace,
                          (cudaStream_t)stream);
}

static void fill_plan(const Layout &L, const TcLaunch &t, hq_plan_info *out) {
  std::memset(out, 0, sizeof(*out));
  out->kernel = t.kind;
  out->layout = L.bs;
  out->token_tile = t.bnt;
  out->weight_tiles = t.ntw;
  out->token_tiles = t.mtiles;
  out->ctas = t.nctas;
}

hq_status hq_gemm_plan(const hq_quant_desc *desc, const hq_compute_config *cfg, int M, int N, int K,
                       hq_plan_info *out) {
  if (!out) return HQ_ERR_INVALID_ARG;
  DensePlan pl;
  const hq_status ps = plan_dense_cfg(desc, cfg, M, N, K, &pl);
  if (ps != HQ_OK) return ps;
  fill_plan(pl.L, pl.s, out);
  return HQ_OK;
}

hq_status hq_moe_plan(const hq_quant_desc *desc, int T, int topk, int E, int N, int K, int a_per_slot,
                      hq_plan_info *out) {
  if (!out) return HQ_ERR_INVALID_ARG;
  MoePlan pl;
  const hq_status ps = plan_moe(desc, T, topk, E, N, K, a_per_slot, &pl);
  if (ps != HQ_OK) return ps;
  fill_plan(pl.L, pl.s, out);
  return HQ_OK;
}

size_t hq_gemm_config_workspace_bytes(const hq_quant_desc *desc, const hq_compute_config *cfg, int M, int N,
                                      int K) {
  DensePlan pl;
  if (plan_dense_cfg(desc, cfg, M, N, K, &pl) != HQ_OK) return 0;
  void *a, *b;
  return dense_ws(pl, M, K, nullptr, &a, &b);
}

size_t hq_gemm_workspace_bytes(const hq_quant_desc *desc, int M, int N, int K) {
  return hq_gemm_config_workspace_bytes(desc, nullptr, M, N, K);
}

hq_status hq_gemm_config(const hq_quant_desc *desc, const hq_compute_config *cfg, int M, int N, int K,
                         const void *packed_w, const void *a, const void *a_scales, const float *a_global,
                         void *c_bf16, void *workspace, size_t ws_bytes, hq_stream_t stream) {
  DensePlan pl;
  const hq_status ps = plan_dense_cfg(desc, cfg, M, N, K, &pl);
  if (ps != HQ_OK) return ps;
  if (M == 0) return HQ_OK;
  const hq_status as = dense_args(pl, packed_w, a, a_scales, a_global, c_bf16);
  if (as != HQ_OK) return as;
  void *split_ws, *a_dec;
  const size_t need = dense_ws(pl, M, K, (uint8_t *)workspace, &split_ws, &a_dec);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return HQ_ERR_WORKSPACE;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  cudaStream_t st = (cudaStream_t)stream;
  if (pl.L.bs != BS_NONE) {
    // block-scaled MMA: the quantised activations go to the tensor core as they are
    return launch_bs_gemm(pl.L, packed_w, 1, a, M, a_scales, 1, pl.afmt == A_NVFP4 ? a_global : nullptr, M, 0,
                          nullptr, nullptr, c_bf16, pl.s, split_ws, a_dec, st);
  }
  if (pl.L.fmt == W_FP8 && pl.afmt == A_FP8) {
    // E4M3 x E4M3 on the FP8 tensor path; per-token x per-channel scales in the epilogue
    return launch_tc_gemm(pl.L, packed_w, a, M, (const float *)a_scales, nullptr, M, 0, 1, nullptr, nullptr, 1, 0,
                          c_bf16, pl.s, split_ws, st, true);
  }
  const void *a_use = a;
  const float *row_scale = nullptr;
  if (pl.afmt != A_BF16) {
    hq_status s = launch_act_decode(pl.afmt, M, K, a, a_scales, nullptr, 1, a_dec, st);
    if (s != HQ_OK) return s;
    a_use = a_dec;
    if (pl.afmt == A_FP8) row_scale = (const float *)a_scales;
  }
  return launch_tc_gemm(pl.L, packed_w, a_use, M, row_scale, pl.afmt == A_NVFP4 ? a_global : nullptr, M, 0, 1,
                        nullptr, nullptr, 1, 0, c_bf16, pl.s, split_ws, st);
}

hq_status hq_gemm(const hq_quant_desc *desc, int M, int N, int K, const void *packed_w, const void *a,
                  const void *a_scales, const float *a_global, void *c_bf16, void *workspace, size_t ws_bytes,
                  hq_stream_t stream) {
  return hq_gemm_config(desc, nullptr, M, N, K, packed_w, a, a_scales, a_global, c_bf16, workspace, ws_bytes,
                        stream);
}

hq_status hq_moe_permute(int T, int topk, int E, const int32_t *topk_ids, int32_t *expert_offsets, int32_t *perm,
                         int32_t *inv_perm, hq_stream_t stream) {
  if (T < 0 || topk < 1 || E < 1 || E > 1024) return HQ_ERR_INVALID_ARG;
  if (!expert_offsets || (T > 0 && (!topk_ids || !perm || !inv_perm))) return HQ_ERR_INVALID_ARG;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  return launch_moe_permute(T, topk, E, topk_ids, expert_offsets, perm, inv_perm, (cudaStream_t)stream);
}

size_t hq_moe_workspace_bytes(hq_moe_mode mode, const hq_quant_desc *desc, int T, int topk, int E, int N, int K,
                              int a_per_slot, int combine) {
  MoePlan pl;
  if (mode != HQ_MOE_GROUPED && mode != HQ_MOE_INDEXED) return 0;
  if (plan_moe(desc, T, topk, E, N, K, a_per_slot, &pl) != HQ_OK) return 0;
  MoeWs w;
  return moe_ws(pl, mode, E, K, N, combine, true, nullptr, &w);
}

hq_status hq_moe_gemm(hq_moe_mode mode, const hq_quant_desc *desc, int T, int topk, int E, int N, int K,
                      const void *packed_w, const void *a, const void *a_scales, const float *a_global,
                      int a_per_slot, const int32_t *topk_ids, const float *topk_weights,
                      const int32_t *expert_offsets, const int32_t *perm, int combine, float routed_scale,
                      void *out_bf16, void *workspace, size_t ws_bytes, hq_stream_t stream) {
  MoePlan pl;
  if (mode != HQ_MOE_GROUPED && mode != HQ_MOE_INDEXED) return HQ_ERR_INVALID_ARG;
  const hq_status ps = plan_moe(desc, T, topk, E, N, K, a_per_slot, &pl);
  if (ps != HQ_OK) return ps;
  if (T == 0) return HQ_OK;
  if (!packed_w || !a || !out_bf16) return HQ_ERR_INVALID_ARG;
  if (!aligned16(packed_w) || !aligned16(a) || !aligned16(out_bf16)) return HQ_ERR_INVALID_ARG;
  const bool routed = expert_offsets && perm;
  if (!routed && (expert_offsets || perm || !topk_ids)) return HQ_ERR_INVALID_ARG;
  if (a_scales) {
    if (pl.afmt == A_BF16 || ((uintptr_t)a_scales & 3u)) return HQ_ERR_INVALID_ARG;
    if (pl.afmt == A_NVFP4 && !a_global) return HQ_ERR_INVALID_ARG;
  }
  if (combine && (!topk_weights || (N % 8) != 0)) return HQ_ERR_INVALID_ARG;
  MoeWs w;
  const size_t need = moe_ws(pl, mode, E, K, N, combine, true, (uint8_t *)workspace, &w);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return HQ_ERR_WORKSPACE;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  cudaStream_t st = (cudaStream_t)stream;
  if (!routed) {
    const hq_status s = launch_moe_permute(T, topk, E, topk_ids, w.r_off, w.r_perm, w.r_inv, st);
    if (s != HQ_OK) return s;
    expert_offsets = w.r_off;
    perm = w.r_perm;
  }
  return moe_run(pl, mode, T, topk, E, N, K, packed_w, a, a_scales, a_global, a_per_slot ? 1 : topk, nullptr,
                 expert_offsets, perm, topk_weights, routed_scale, combine, out_bf16, w, st);
}

size_t hq_moe_gated_workspace_bytes(hq_moe_mode mode, const hq_quant_desc *desc, int T, int topk, int E, int I,
                                    int K) {
  if (I < 1 || (I % (TILE_N / 2)) != 0 || I > (1 << 29)) return 0;
  return hq_moe_workspace_bytes(mode, desc, T, topk, E, 2 * I, K, 0, 0);
}

hq_status hq_moe_gemm_gated(hq_moe_mode mode, const hq_quant_desc *desc, int T, int topk, int E, int I, int K,
                            const void *packed_w, const void *a, const void *a_scales, const float *a_global,
                            const int32_t *topk_ids, const int32_t *expert_offsets, const int32_t *perm,
                            void *out_bf16, void *workspace, size_t ws_bytes, hq_stream_t stream) {
  MoePlan pl;
  if (mode != HQ_MOE_GROUPED && mode != HQ_MOE_INDEXED) return HQ_ERR_INVALID_ARG;
  if (I < 1 || (I % (TILE_N / 2)) != 0 || I > (1 << 29)) return HQ_ERR_INVALID_ARG;
  const int N = 2 * I;
  const hq_status ps = plan_moe(desc, T, topk, E, N, K, 0, &pl);
  if (ps != HQ_OK) return ps;
  pl.L.gated = 1;  // weights from hq_pack_weights_gated; the epilogue writes silu(gate) * up
  if (T == 0) return HQ_OK;
  if (!packed_w || !a || !out_bf16) return HQ_ERR_INVALID_ARG;
  if (!aligned16(packed_w) || !aligned16(a) || !aligned16(out_bf16)) return HQ_ERR_INVALID_ARG;
  const bool routed = expert_offsets && perm;
  if (!routed && (expert_offsets || perm || !topk_ids)) return HQ_ERR_INVALID_ARG;
  if (a_scales) {
    if (pl.afmt == A_BF16 || ((uintptr_t)a_scales & 3u)) return HQ_ERR_INVALID_ARG;
    if (pl.afmt == A_NVFP4 && !a_global) return HQ_ERR_INVALID_ARG;
  }
  MoeWs w;
  const size_t need = moe_ws(pl, mode, E, K, N, 0, true, (uint8_t *)workspace, &w);
  if (!workspace || ws_bytes < need || !aligned16(workspace)) return HQ_ERR_WORKSPACE;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  cudaStream_t st = (cudaStream_t)stream;
  if (!routed) {
    const hq_status s = launch_moe_permute(T, topk, E, topk_ids, w.r_off, w.r_perm, w.r_inv, st);
    if (s != HQ_OK) return s;
    expert_offsets = w.r_off;
    perm = w.r_perm;
  }
  return moe_run(pl, mode, T, topk, E, N, K, packed_w, a, a_scales, a_global, topk, nullptr, expert_offsets, perm,
                 nullptr, 1.f, 0, out_bf16, w, st);
}

size_t hq_moe_masked_workspace_bytes(const hq_quant_desc *desc, int E, int slab, int N, int K, int expected_m) {
  MoePlan pl;
  if (plan_moe_masked(desc, E, slab, N, K, expected_m, &pl) != HQ_OK) return 0;
  MoeWs w;
  Carver c{nullptr};
  c.off = moe_ws(pl, HQ_MOE_GROUPED, E, K, N, 0, false, nullptr, &w);
  c.take((size_t)(E + 1) * sizeof(int32_t));
  c.take((size_t)E * slab * sizeof(int32_t));
  return c.off;
}

hq_status hq_moe_gemm_masked(const hq_quant_desc *desc, int E, int slab, int N, int K, const void *packed_w,
                             const void *a_bf16, const int32_t *expert_num_tokens, int expected_m, void *out_bf16,
                             void *workspace, size_t ws_bytes, hq_stream_t stream) {
  MoePlan pl;
  const hq_status ps = plan_moe_masked(desc, E, slab, N, K, expected_m, &pl);
  if (ps != HQ_OK) return ps;
  if (!packed_w || !a_bf16 || !expert_num_tokens || !out_bf16) return HQ_ERR_INVALID_ARG;
  if (!aligned16(packed_w) || !aligned16(a_bf16) || !aligned16(out_bf16)) return HQ_ERR_INVALID_ARG;
  MoeWs w;
  Carver c{(uint8_t *)workspace};
  c.off = moe_ws(pl, HQ_MOE_GROUPED, E, K, N, 0, false, (uint8_t *)workspace, &w);
  int32_t *offsets = (int32_t *)c.take((size_t)(E + 1) * sizeof(int32_t));
  int32_t *perm = (int32_t *)c.take((size_t)E * slab * sizeof(int32_t));
  if (!workspace || ws_bytes < c.off || !aligned16(workspace)) return HQ_ERR_WORKSPACE;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  cudaStream_t st = (cudaStream_t)stream;
  const hq_status s = launch_moe_masked_prepare(E, slab, expert_num_tokens, offsets, perm, st);
  if (s != HQ_OK) return s;
  // every valid row is its own slot: one row per slot (div = 1), no combine
  return moe_run(pl, HQ_MOE_GROUPED, E * slab, 1, E, N, K, packed_w, a_bf16, nullptr, nullptr, 1, expert_num_tokens,
                 offsets, perm, nullptr, 1.f, 0, out_bf16, w, st);
}

hq_status hq_silu_and_mul(int R, int I, const void *y_bf16, void *out_bf16, hq_stream_t stream) {
  if (R < 0 || I < 8 || (I % 8) != 0) return HQ_ERR_INVALID_ARG;
  if (R == 0) return HQ_OK;
  if (!y_bf16 || !out_bf16 || !aligned16(y_bf16) || !aligned16(out_bf16)) return HQ_ERR_INVALID_ARG;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  return launch_silu_and_mul(R, I, y_bf16, out_bf16, (cudaStream_t)stream);
}

hq_status hq_moe_unpermute_sum(int T, int topk, int N, const void *y_bf16, const int32_t *inv_perm,
                               const float *topk_weights, float routed_scale, void *out_bf16, hq_stream_t stream) {
  if (T < 0 || topk < 1 || N < 8 || (N % 8) != 0) return HQ_ERR_INVALID_ARG;
  if (T == 0) return HQ_OK;
  if (!y_bf16 || !topk_weights || !out_bf16 || !aligned16(y_bf16) || !aligned16(out_bf16)) return HQ_ERR_INVALID_ARG;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  return launch_unpermute_sum(T, topk, N, y_bf16, inv_perm, topk_weights, routed_scale, out_bf16,
                              (cudaStream_t)stream);
}

}  // extern "C"
