// Block-circulant layer kernels for block size p = 4096 (one translation unit per p).
#include "circ_kernels.cuh"

namespace rdfft {
RDFFT_CIRC_INSTANCE(4096)
}  // namespace rdfft
