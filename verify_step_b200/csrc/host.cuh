// Host-side helpers shared by the entry points (defined in abi.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <mutex>
#include <utility>

#include "../../include/sd_verify.h"

namespace sdv {

// Cache of a __device__ variable's address per device, keyed on the CUDA context it was
// looked up in (a device reset invalidates addresses; the next lookup then repeats).
struct SymbolSlot {
  static constexpr int kDevices = 64;
  std::mutex mu;
  void *addr[kDevices] = {};
  void *ctx[kDevices] = {};
};

// Device address of ``symbol`` (a __device__ variable of this library) on the current device,
// looked up with cudaGetSymbolAddress when the cache has none for the current context.  A
// symbol's host-side name is not a device address, so kernels get this value instead.
// nullptr if it cannot be obtained.
void *symbol_address(SymbolSlot &slot, const void *symbol);

// Device address of the current device's status word (nullptr if it cannot be obtained).
int *device_status_word();

// Streaming multiprocessors of the current device (0 on failure).
int sm_count();

// 2D bf16 tensor map over a row-major matrix [outer, inner] with the given row stride in
// bytes, box [box_outer, box_inner], 128-byte swizzle (or none), zero fill out of bounds.
bool encode_tmap_2d_bf16(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                         uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer,
                         bool swizzle128 = true);

// A [rows x D] bf16 matrix viewed as (64 columns, rows, D / 64 chunks), so that one 3D box of
// box_rows rows brings all of a row block's column chunks at once, chunk-major with the 128-byte
// swizzle (the layout of box_rows x 64 2D boxes stored one after another).  False if the driver
// refuses the view.
bool encode_tmap_kv_chunks_bf16(CUtensorMap *map, const void *base, uint64_t D, uint64_t rows,
                                uint32_t box_rows);

inline sd_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SD_OK : SD_ERR_CUDA; }

// Programmatic dependent launch: off unless the environment sets SDV_PDL=1 (read once per
// process).  Every kernel calls pdl_wait() before its first global access, so either way is
// correct; on the spec step the plain stream order measured faster.
bool pdl_enabled();

// Launches ``kernel`` with programmatic stream serialization (the kernel must call pdl_wait()
// before touching global memory written by earlier work in the stream).
template <typename... KArgs, typename... Args>
inline cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace sdv
