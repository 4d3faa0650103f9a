// Host-side construction of TMA tensor maps. The driver entry point is looked
// up through the runtime, so the library needs no link against libcuda.
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace sa {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 tensor [BH][T][Hh][Ww][d] (natural video order, d innermost) seen as a
// 5-D TMA tensor whose box is one 64-channel slice of a block: pt*frames
// consecutive frames of a ph x pw spatial patch (pt*frames*ph*pw token rows of
// 128 bytes, frame-major, then row-major inside the patch), written to shared
// memory with the 128-byte swizzle. Coordinates are (channel, w, h, t, bh).
inline bool encode_tile_map(CUtensorMap* map, const void* base, int BH, int T, int Hh, int Ww,
                            int d, int pt, int ph, int pw, int frames = 1) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[5] = {cuuint64_t(d), cuuint64_t(Ww), cuuint64_t(Hh), cuuint64_t(T),
                        cuuint64_t(BH)};
  cuuint64_t row = cuuint64_t(d) * 2;
  cuuint64_t strides[4] = {row, row * Ww, row * Ww * Hh, row * Ww * Hh * T};
  cuuint32_t box[5] = {64, cuuint32_t(pw), cuuint32_t(ph), cuuint32_t(pt * frames), 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The square patch of one frame: encode_tile_map with the block (1, P, P).
inline bool encode_patch_map(CUtensorMap* map, const void* base, int BH, int T, int Hh, int Ww,
                             int d, int P, int frames = 1) {
  return encode_tile_map(map, base, BH, T, Hh, Ww, d, 1, P, P, frames);
}

// fp32 matrix [rows][cols] (cols innermost, cols * 4 a multiple of 16 bytes)
// seen as a 2-D TMA tensor whose box is 32 columns (128 bytes) x box_rows
// rows, written to shared memory with the 128-byte swizzle; rows or columns
// past the end read as zeros. Coordinates are (column, row).
inline bool encode_rows_f32(CUtensorMap* map, const void* base, long long rows, int cols,
                            int box_rows) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols) * 4};
  cuuint32_t box[2] = {32, cuuint32_t(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace sa
