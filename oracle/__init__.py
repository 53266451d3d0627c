"""Float64 CPU oracle for rdFFT and the block-circulant layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or run
anything in this package: only tests/, the package smoke check in
__graft_entry__.smoke() and bench.py's CPU-baseline leg use it. It shares no code
with the CUDA path (no kernels, headers, tables or helpers); both sides only draw
their inputs from the `synthetic` module.

What it computes, each function from its plain definition (no FFT, no blocking,
no reordering beyond the definition):

* dft_packed / idft_packed -- the O(p^2) real DFT of each row, written into the
  packed real layout of "Memory-Efficient Training with In-Place FFT
  Implementation" (summary page, "Approach"; paper-notes page, method section,
  "Squeeze N+2 -> N"): y_0 at index 0, y_{p/2} at index p/2, Re y_k at index k and
  Im y_k at index p-k for 0 < k < p/2.
* circulant_matrix / circ_forward / circ_backward -- the block-circulant linear
  layer as a dense D x D matrix built from its q x q circulant blocks (paper-notes
  page, method section, "Circulant matrix training adaptation"), with grad_x the
  transposed product and grad_c the chain rule through the matrix entries.
* packed_to_rfft / rfft_to_packed -- the cast between a packed row and its explicit
  complex bins Y_0..Y_{p/2} (summary page, "Limitations").
* dft2_packed / unpack2_spectrum / idft2_packed -- the 2-D real DFT of an R x C
  image by its definition (two DFT matrices), written into the per-axis packed
  layout documented in dft2_packed (paper-notes page, "Limitations and outlook"
  leaves 2-D open; that layout is the reading taken); dft2_packed_at gives single
  slots of it by the definition, for images too large for the matrix form.

Every function here is pinned by tests/test_oracle_pins.py against closed forms,
invariants, a library FFT on the special cases that reduce to it, hand values and
finite differences. No function is "parity unpinned".
"""
from .rdfft_oracle import (  # noqa: F401
    dft_packed,
    idft_packed,
    unpack_spectrum,
    circulant_matrix,
    circ_forward,
    circ_backward,
    packed_to_rfft,
    rfft_to_packed,
    dft2_full,
    dft2_packed,
    dft2_packed_at,
    unpack2_spectrum,
    idft2_packed,
)
