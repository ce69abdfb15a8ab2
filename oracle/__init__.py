"""Plain float64 CPU oracle for the fused Hadamard rotation + quantization path.

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports, links or calls this
package; only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code,
table or constant generator with the CUDA path.

What it computes, and where the pages define it:

* ``sylvester_hadamard`` / ``rotate`` -- the deterministic Sylvester Hadamard
  matrix built by the doubling H -> [[H, H], [H, -H]] and normalised by the
  square root of its size ("Rotation Transform", AutoRound docs, section 1.5
  "Deterministic vs random Hadamard"), applied to every row as a dense
  float64 product, full-size or block-diagonal with ``rotation_size`` /
  ``block_size`` blocks (same page, sections 1.2 and 2.1).  The orthogonality
  the page states in its introduction (R @ R^T = I) is what lets the rotated
  activations meet pre-rotated weights.
* ``paley_hadamard`` / ``hadamard_matrix`` -- the non-power-of-2 sizes of
  the same section 1.5: n = K * 2^m combines a base Hadamard matrix of order
  K with a Sylvester block.  The pages print no base matrix; the reading is
  Paley's second construction (a published method, cited on the function)
  and the Kronecker product H_K (x) H_(2^m).
* ``random_hadamard_matrix`` / ``rotate_signed`` -- the random Hadamard
  matrix H @ diag(+/-1) / sqrt(N) of the same section 1.5 (signs persisted as
  int8, section 1.7), and its transpose diag(+/-1) @ H / sqrt(N), which is its
  inverse and puts the signs ahead of the transform as in orbitquant's RPBH
  ("orbitquant 0.2.0", how it works).
* ``rpbh_rotate`` / ``sphere_lloyd_max`` / ``quantize_codebook`` -- the
  orbitquant method ("orbitquant 0.2.0", Method Conformance): RPBH rotation
  (permutation, Rademacher signs, block FWHT, orthonormal scaling) and the
  online quantizer (per-token norm, normalized rotation, nearest centroid of
  the unit-sphere Lloyd-Max codebook, rescaling).  Readings on each function.
* ``quantize_int4_sym`` / ``quantize_int8_per_token`` -- round-to-nearest
  with symmetric range (the RTN proxy with wbits / groupsize / sym of
  "Pre-Process (Rotation Preprocessing)", OneCompression docs, Workflow note).
* ``quantize_mxfp4`` -- the MXFP4 scheme the rotation targets ("Rotation
  Transform", introduction and section 2.1: MX block 32).  The pages do not
  define the format's internals; the reading used is the OCP MX v1.0 rule
  (E2M1 elements, E8M0 shared scale, floor-based exponent).

* ``quantize_nvfp4`` -- the NVFP4 scheme (same page, introduction and section
  2.1: block 16); the pages give no encoding, the reading used is NVIDIA's
  public NVFP4 definition (E2M1 elements, an FP8 E4M3 scale per 16 elements,
  an optional per-tensor fp32 scale).

Readings of points the pages leave open (rounding half to even, the fp16 scale
used for the codes, the symmetric +/-7 / +/-127 range, zero groups, nibble
order, non-finite scales) are stated on each function.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
to values the pages or the mathematics fix (hand cases, closed forms, library
routines, invariants).  End-to-end rotated-and-quantized values have no worked
example on the pages; they are pinned only through their pinned parts.
"""

from .hadq_oracle import (  # noqa: F401
    E2M1_GRID,
    INT4_QMAX,
    INT8_QMAX,
    MX_GROUP,
    NV_GROUP,
    E4M3_MAX,
    codes_with_scale,
    e2m1_encode,
    e4m3_encode,
    e8m0_exponent,
    fp16_scale_midpoint_distance,
    hadamard_matrix,
    jacobsthal,
    paley_hadamard,
    PALEY_FIELDS,
    quadratic_character,
    split_size,
    pack_codes,
    pack_nibbles,
    quantize_codebook,
    rpbh_inverse,
    rpbh_rotate,
    sphere_lloyd_max,
    sphere_marginal_cdf,
    sphere_partial_first_moment,
    quantize,
    quantize_int4_sym,
    quantize_int8_per_token,
    quantize_mxfp4,
    quantize_nvfp4,
    random_hadamard_matrix,
    resolve_block,
    rotate,
    rotate_quant,
    rotate_quant_signed,
    rotate_signed,
    round_to_binary,
    sign_vector,
    sylvester_hadamard,
    to_bf16_bits,
    to_fp16,
    to_e4m3,
    to_fp32,
)
