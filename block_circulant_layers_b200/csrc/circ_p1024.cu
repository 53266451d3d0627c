// Block-circulant layer kernels for block size p = 1024 (one translation unit per p).
#include "circ_kernels.cuh"

namespace rdfft {
RDFFT_CIRC_INSTANCE(1024)
}  // namespace rdfft
