// Block-circulant layer kernels for block size p = 2048 (one translation unit per p).
#include "circ_kernels.cuh"

namespace rdfft {
RDFFT_CIRC_INSTANCE(2048)
}  // namespace rdfft
