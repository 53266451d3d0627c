// Block-circulant layer kernels for block size p = 256 (one translation unit per p).
#include "circ_kernels.cuh"

namespace rdfft {
RDFFT_CIRC_INSTANCE(256)
}  // namespace rdfft
