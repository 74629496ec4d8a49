// Library-wide host helpers and the status entry points of the C ABI.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "host.cuh"

namespace sdv {

// Per-device status word: kernels record the first device-side error here.
__device__ int g_status_word;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

static CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

void *symbol_address(SymbolSlot &slot, const void *symbol) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= SymbolSlot::kDevices)
    return nullptr;
  // The context the address belongs to: a device reset or a new primary context makes a cached
  // address stale, so the cache is keyed on the context that is current now.
  CUcontext ctx = nullptr;
  CtxGetCurrentFn get = ctx_get_current_fn();
  if (get == nullptr || get(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  std::lock_guard<std::mutex> lock(slot.mu);
  if (slot.addr[dev] == nullptr || ctx == nullptr || slot.ctx[dev] != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) return nullptr;
    slot.addr[dev] = p;
    slot.ctx[dev] = ctx;
  }
  return slot.addr[dev];
}

int *device_status_word() {
  static SymbolSlot slot;
  return reinterpret_cast<int *>(symbol_address(slot, &g_status_word));
}

bool pdl_enabled() {
  static const bool on = [] {
    const char *e = getenv("SDV_PDL");
    return e && strcmp(e, "1") == 0;
  }();
  return on;
}

// One thread waits on a barrier no one arrives at: the bounded wait must give up and report.
__global__ void selftest_wait_kernel(int *status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  pdl_wait();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag)) record_status(status, SD_ERR_TIMEOUT);
}

int sm_count() {
  static int cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool encode_tmap_2d_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                         uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                         bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_kv_chunks_bf16(CUtensorMap *map, const void *base, uint64_t D, uint64_t rows,
                                uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || D % 64) return false;
  // (64 columns, rows, D / 64 column chunks): one box = box_rows rows of every chunk, laid
  // out chunk-major in shared memory, each chunk's rows 128 bytes with the 128-byte swizzle
  const cuuint64_t dims[3] = {64, rows, D / 64};
  const cuuint64_t strides[2] = {D * 2, 128};
  const cuuint32_t box[3] = {64, box_rows, (cuuint32_t)(D / 64)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace sdv

extern "C" {

const char *sd_status_string(sd_status s) {
  switch (s) {
    case SD_OK: return "ok";
    case SD_ERR_INVALID_ARG: return "invalid argument";
    case SD_ERR_UNSUPPORTED: return "unsupported configuration";
    case SD_ERR_WORKSPACE: return "workspace too small";
    case SD_ERR_CUDA: return "CUDA error";
    case SD_ERR_TIMEOUT: return "device wait timed out";
    case SD_ERR_DEVICE: return "out-of-range index on the device";
  }
  return "unknown status";
}

sd_status sd_device_status_read(int *out, sd_stream stream) {
  if (!out) return SD_ERR_INVALID_ARG;
  int *w = sdv::device_status_word();
  if (!w) return SD_ERR_CUDA;
  if (cudaMemcpyAsync(out, w, sizeof(int), cudaMemcpyDeviceToHost, (cudaStream_t)stream) !=
      cudaSuccess)
    return SD_ERR_CUDA;
  return sdv::cuda_status(cudaStreamSynchronize((cudaStream_t)stream));
}

sd_status sd_device_status_clear(sd_stream stream) {
  int *w = sdv::device_status_word();
  if (!w) return SD_ERR_CUDA;
  return sdv::cuda_status(cudaMemsetAsync(w, 0, sizeof(int), (cudaStream_t)stream));
}

sd_status sd_selftest_bounded_wait(sd_stream stream) {
  int *w = sdv::device_status_word();
  if (!w) return SD_ERR_CUDA;
  return sdv::cuda_status(sdv::launch(sdv::selftest_wait_kernel, dim3(1), dim3(32), 0,
                                      (cudaStream_t)stream, w));
}

int sd_version(void) { return 100; }

}  // extern "C"
