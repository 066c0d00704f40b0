// tcgen05 (5th-generation tensor core) GEMMs of libspectra: the encode
// projection C = H W_down and the calibration Gram G = H^T H.
#include "kernels.h"

namespace spectra {

cudaError_t launch_project_tcgen05(const CodecDev&, const uint16_t*, const uint16_t*, int, float*,
                                   int64_t, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t launch_gram_tcgen05(const uint16_t*, int64_t, int, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace spectra
