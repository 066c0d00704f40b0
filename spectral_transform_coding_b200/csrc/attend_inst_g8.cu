// Instantiations of the decode attention kernel for groups of 8 coordinates
// (split from the host code so that the variants compile in parallel).
#include "attend_kernel.cuh"

namespace spectra {
namespace attend {

AttendKernel attend_kernel_ptr_g8(int NT, int CH, int MV) {
  const int key = NT * 100 + CH * 10 + MV;
  switch (key) {
    case 122: return attend_kernel<8, 1, 2, 2>;
    case 124: return attend_kernel<8, 1, 2, 4>;
    case 128: return attend_kernel<8, 1, 2, 8>;
    case 142: return attend_kernel<8, 1, 4, 2>;
    case 144: return attend_kernel<8, 1, 4, 4>;
    case 148: return attend_kernel<8, 1, 4, 8>;
    case 222: return attend_kernel<8, 2, 2, 2>;
    case 224: return attend_kernel<8, 2, 2, 4>;
    case 228: return attend_kernel<8, 2, 2, 8>;
    case 242: return attend_kernel<8, 2, 4, 2>;
    case 244: return attend_kernel<8, 2, 4, 4>;
    case 248: return attend_kernel<8, 2, 4, 8>;
    case 182: return attend_kernel<8, 1, 8, 2>;
    case 184: return attend_kernel<8, 1, 8, 4>;
    case 188: return attend_kernel<8, 1, 8, 8>;
    default: return nullptr;
  }
}

}  // namespace attend
}  // namespace spectra
