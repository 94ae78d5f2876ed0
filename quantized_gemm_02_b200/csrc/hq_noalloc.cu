// hq_gemm_noalloc: the dense GEMM for callers that cannot allocate device
// memory.
//
// Some callers cannot call cudaMalloc at the point where they run a GEMM:
// custom allocator hooks and embedded runtimes that own all device memory and
// forbid side allocations, plugins loaded into a host framework that gives
// them no allocator at all, and code paths that must not allocate while they
// run.  hq_gemm needs a caller-supplied workspace (split-K
// partial sums, tile counters, decoded activations).  This entry point instead
// uses one fixed scratch array that lives in the library's own device image:
// a file-scope __device__ array that every GPU loading the library holds
// until the process exits.
//
// Host code must not hand the array's name to a kernel: in host code that
// name is a host-side stand-in, not a device address.  The address is
// obtained with cudaGetSymbolAddress, once per device, with that device
// current, and cached.
#include "hq_internal.cuh"

namespace hq {

// Maximum scratch a single hq_gemm_noalloc call may use (64 MiB).
constexpr size_t NOALLOC_SCRATCH_BYTES = (size_t)64 << 20;

__device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

static void *g_noalloc_ptr[64];  // device address of g_noalloc_scratch, per device ordinal

static hq_status noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
  if (dev < 0 || dev >= 64) return HQ_ERR_CUDA;
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return HQ_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return HQ_OK;
}

}  // namespace hq

extern "C" hq_status hq_gemm_noalloc(const hq_quant_desc *desc, int M, int N, int K, const void *packed_w,
                                     const void *a, const void *a_scales, const float *a_global, void *c_bf16,
                                     hq_stream_t stream) {
  using namespace hq;
  DensePlan pl;
  const hq_status ps = plan_dense(desc, M, N, K, &pl);
  if (ps != HQ_OK) return ps;
  if (M == 0) return HQ_OK;
  void *split_ws, *a_dec;
  const size_t need = dense_ws(pl, M, K, nullptr, &split_ws, &a_dec);
  if (need > NOALLOC_SCRATCH_BYTES) return HQ_ERR_WORKSPACE;
  // every argument check hq_gemm makes, before anything is enqueued
  const hq_status as = dense_args(pl, packed_w, a, a_scales, a_global, c_bf16);
  if (as != HQ_OK) return as;
  if (!device_is_sm100()) return HQ_ERR_ARCH;
  void *scratch = nullptr;
  const hq_status ss = noalloc_scratch(&scratch);
  if (ss != HQ_OK) return ss;
  // The array keeps the previous call's contents; the split-K tile counters
  // at its head must start at zero.
  {
    if (cudaMemsetAsync(scratch, 0, tc_counter_bytes(pl.s), (cudaStream_t)stream) != cudaSuccess) return HQ_ERR_CUDA;
  }
  return hq_gemm(desc, M, N, K, packed_w, a, a_scales, a_global, c_bf16, scratch, NOALLOC_SCRATCH_BYTES, stream);
}
