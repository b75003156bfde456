// Fused decode kernels for prod key caches: one instantiation per (index bits, value bits)
// and block shape (see decode_kernel.cuh).
#include "decode_kernel.cuh"

namespace tq {
namespace dec {

tq_status launch_kind_prod(const DecodeArgs& a, int mb, int vb, dim3 grid, int max_heads,
                           bool two, bool pdl, cudaStream_t st) {
  switch (mb * 8 + vb) {
    case 1 * 8 + 0: return run_decode_shape<1, 0, kProd>(a, grid, max_heads, two, pdl, st);
    case 1 * 8 + 2: return run_decode_shape<1, 2, kProd>(a, grid, max_heads, two, pdl, st);
    case 1 * 8 + 4: return run_decode_shape<1, 4, kProd>(a, grid, max_heads, two, pdl, st);
    case 2 * 8 + 0: return run_decode_shape<2, 0, kProd>(a, grid, max_heads, two, pdl, st);
    case 2 * 8 + 2: return run_decode_shape<2, 2, kProd>(a, grid, max_heads, two, pdl, st);
    case 2 * 8 + 4: return run_decode_shape<2, 4, kProd>(a, grid, max_heads, two, pdl, st);
    case 3 * 8 + 0: return run_decode_shape<3, 0, kProd>(a, grid, max_heads, two, pdl, st);
    case 3 * 8 + 2: return run_decode_shape<3, 2, kProd>(a, grid, max_heads, two, pdl, st);
    case 3 * 8 + 4: return run_decode_shape<3, 4, kProd>(a, grid, max_heads, two, pdl, st);
    default: return TQ_EUNSUPPORTED;
  }
}

}  // namespace dec
}  // namespace tq
