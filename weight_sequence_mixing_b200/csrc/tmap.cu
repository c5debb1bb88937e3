// Host-side construction of TMA tensor maps (driver entry point resolved at
// run time through the runtime, so the library does not link libcuda directly).
#include "tc_gemm.cuh"

namespace ttt {

PFN_tmapEncodeTiled tmap_encoder() {
  static PFN_tmapEncodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_tmapEncodeTiled>(p);
  }
  return fn;
}

int current_device() {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess ? dev : -1;
}

int sm_count() {
  static IntPerDevice counts;
  const int dev = current_device();
  return counts.get(dev, [dev] {
    int n = 0;
    if (dev < 0 || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;  // a B200's count, if the device cannot be asked
    return n;
  });
}

bool make_tmap(CUtensorMap* out, const void* base, int eb, int64_t cols, int64_t rows, int64_t batches,
               int64_t row_pitch_elems, int64_t batch_pitch_elems, int box_rows) {
  return make_tmap_ex(out, base, eb, cols, rows, batches, row_pitch_elems, batch_pitch_elems, 128 / eb, box_rows, 128);
}

bool make_tmap_ex(CUtensorMap* out, const void* base, int eb, int64_t cols, int64_t rows, int64_t batches,
                  int64_t row_pitch_elems, int64_t batch_pitch_elems, int box_cols, int box_rows, int swizzle) {
  PFN_tmapEncodeTiled enc = tmap_encoder();
  if (!enc || !base) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0) return false;
  if (cols <= 0 || rows <= 0 || batches <= 0) return false;
  if (((row_pitch_elems * eb) & 15) != 0 || ((batch_pitch_elems * eb) & 15) != 0) return false;
  if (box_rows <= 0 || box_rows > 256 || box_cols <= 0 || box_cols * eb > swizzle) return false;
  if (((box_cols * eb) & 15) != 0) return false;
  const CUtensorMapSwizzle sw = swizzle == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (swizzle != 128 && swizzle != 64 && swizzle != 32) return false;
  const CUtensorMapDataType dt = eb == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(batches)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(row_pitch_elems * eb),
                           static_cast<cuuint64_t>(batch_pitch_elems * eb)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(out, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace ttt
