// api.cu -- status strings, version, plan sizing and the tensor-map encoder
// shared by the kernels' host code.
#include <cudaTypedefs.h>
#include <math.h>

#include "internal.h"

namespace svoo {

CUresult encode_tiled_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows, uint32_t box_cols) {
  // looked up once; a function-local static is initialised exactly once even
  // when several host threads make their first call at the same time
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  if (!fn) return CUDA_ERROR_NOT_FOUND;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace svoo

using namespace svoo;

extern "C" const char* svoo_status_string(svoo_status s) {
  switch (s) {
    case SVOO_OK: return "ok";
    case SVOO_ERR_INVALID_ARG: return "invalid argument";
    case SVOO_ERR_WORKSPACE: return "workspace too small";
    case SVOO_ERR_UNSUPPORTED: return "unsupported configuration";
    case SVOO_ERR_CUDA: return "CUDA launch or runtime error";
    case SVOO_ERR_TIMEOUT: return "device wait timed out";
    case SVOO_ERR_INTERNAL: return "internal error";
  }
  return "unknown status";
}

extern "C" int svoo_version(void) { return (0 << 16) | 1; }

extern "C" svoo_status svoo_plan_counts(const svoo_shape* shape, int n_qc, int n_kc, int block_q,
                                        int64_t counts[12]) {
  if (!shape_ok(shape) || !counts) return SVOO_ERR_INVALID_ARG;
  if (n_qc < 1 || n_qc > 256 || n_kc < 1 || n_kc > 256) return SVOO_ERR_INVALID_ARG;
  if (block_q != 64 && block_q != 128) return SVOO_ERR_INVALID_ARG;
  const int64_t BH = bh_of(shape), N = shape->N;
  const int64_t Gq = groups_q(shape, n_qc), Gk = groups_k(shape, n_kc), W = mask_words(shape, n_kc);
  counts[0] = BH * Gq * W;                              // kmask (uint64)
  counts[1] = BH * N;                                   // q_label
  counts[2] = BH * Gq;                                  // q_sizes
  counts[3] = BH * 8;                                   // stats
  counts[4] = BH * N;                                   // q_perm
  counts[5] = BH * (Gq + 1);                            // q_off
  counts[6] = BH * N;                                   // k_perm
  counts[7] = BH * (Gk + 1);                            // k_off
  counts[8] = BH * tile_cap(shape, n_qc, block_q) * 4;  // tiles
  counts[9] = BH;                                       // tile_count
  counts[10] = BH * unit_cap(shape, n_qc) * 4;          // units
  counts[11] = BH;                                      // unit_count
  return SVOO_OK;
}

// SNR-guided top-p schedule (iCATS section 4.2 and appendix A: top-p of each
// denoising call from a smooth function of log SNR, computed offline; dense
// before the first sparse call). With the flow-matching noise level sigma of
// a call, SNR = ((1 - sigma) / sigma)^2 and 1 / (1 + SNR) =
// sigma^2 / (sigma^2 + (1 - sigma)^2), the share of the noise in the signal
// plus noise power, which is a logistic function of log SNR: the budget is
// flat at both ends and falls fastest where SNR = 1.
extern "C" svoo_status svoo_snr_top_p(int steps, int warmup, double p_min, double tau, double shift,
                                      float* p) {
  if (steps < 1 || warmup < 0 || !p) return SVOO_ERR_INVALID_ARG;
  if (!(p_min >= 0.0) || !(tau >= p_min) || !(tau <= 1.0) || !(shift > 0.0) || !isfinite(shift))
    return SVOO_ERR_INVALID_ARG;
  for (int t = 0; t < steps; ++t) {
    if (t < warmup) {
      p[t] = 1.0f;
      continue;
    }
    const double s = 1.0 - static_cast<double>(t) / steps;           // unshifted noise level
    const double sig = shift * s / (1.0 + (shift - 1.0) * s);          // shifted (flow matching)
    const double noise = sig * sig, signal = (1.0 - sig) * (1.0 - sig);
    const double share = noise / (noise + signal);
    p[t] = static_cast<float>(p_min + (tau - p_min) * share);
  }
  return SVOO_OK;
}
