// Host-side helpers shared by the tensor-core kernels: TMA descriptor
// encoding (driver entry point fetched through the runtime, no libcuda link)
// and a per-device cache of the SM count and of one-time kernel attributes.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 [outer, inner] row-major, box (64 inner, box_outer), 128-B swizzle.
inline bool map_rows(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                     uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 3-D bf16 weights [E, K, N] (N contiguous), box (64 N, 64 K, 1), 128-B swizzle.
inline bool map_weights(CUtensorMap* m, const void* base, uint64_t E, uint64_t K, uint64_t N) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {N, K, E};
  cuuint64_t strides[2] = {N * 2, K * N * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 2-D rows [outer, inner] for tile::gather4: box (128 bytes of inner, 1 row),
// 128-B swizzle (4 gathered rows land as 4 rows of a swizzled K-major tile).
inline bool map_rows_gather(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                            bool e4m3) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const uint64_t elem = e4m3 ? 1 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * elem};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem), 1};
  cuuint32_t es[2] = {1, 1};
  return enc(m, e4m3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
             const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D e4m3 codes [outer, inner] row-major, box (128 inner, box_outer), 128-B swizzle.
inline bool map_rows_e4m3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                          uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {128, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// 3-D e4m3 weights stored K-major, codes [E, N, K] (K contiguous), box
// (128 K, box_rows N, 1), 128-B swizzle: a tile lands as box_rows rows of 128 B.
inline bool map_weights_e4m3(CUtensorMap* m, const void* base, uint64_t E, uint64_t N,
                             uint64_t K, uint32_t box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {K, N, E};
  cuuint64_t strides[2] = {K, N * K};
  cuuint32_t box[3] = {128, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Launch `kern` on `s` with programmatic stream serialization: the kernel may
// begin while the previous kernel of the stream finishes (it must call
// grid_dep_wait() before reading that kernel's results).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// attr_set slots: 0-2 grouped GEMM (1 CTA), 3-6 router GEMM, 7-8 grouped GEMM (CTA pair),
// 9-10 CTA-pair GEMM on e4m3 operands, 11-13 grouped GEMM on e4m3 operands,
// 14-15 CTA-pair GEMM with expert tails (its gathering instance 30)
// (+16: the gathering instance of a grouped GEMM slot's kernel, +32: the
// scattering one); 19-22 router GEMM with the top-k epilogue (the router
// kernels have no gathering instance, so 3-6 + 16 is free for them)
struct DeviceInfo {
  int sms = 0;
  bool attr_set[48] = {};
};
inline DeviceInfo g_dev[64];

inline cudaError_t device_info(DeviceInfo** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  DeviceInfo& di = g_dev[dev];
  if (di.sms == 0) {
    err = cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
  }
  *out = &di;
  return cudaSuccess;
}

}  // namespace moe
