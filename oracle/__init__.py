"""Plain fp64 CPU oracle of the rotate-then-quantize path -- TEST INFRASTRUCTURE ONLY.

This package exists to prove the CUDA path right.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import it.  The product package (``rotation_bit_ptq_b200``)
never imports it, and it imports nothing from the product: the two share no
code, tables or constants.  Every step is written the slow, obvious way
(dense matrices, numpy fp64, library sort/search) so that a reader can check
it against the source pages by eye.

Source pages, cited by title and section:

* OrbitQuant -- the OrbitQuant write-up at hotelren.com/news/3376620 (its HTML
  title is unrelated scrape debris).  Sections: 1 (why a fixed N(0,1/d) target
  distribution removes calibration), 2.1 (offline weight quantisation), 2.2
  (online activation quantisation and the cancellation of the rotation), 2.3
  (the RPBH transform), 4.2 (per-d Lloyd-Max codebooks), 6.1/6.3 (debugging
  and cross-platform consistency advice).
* INT8-convrot -- "INT8旋转量化是什么？图像生成模型轻量化全解",
  cloud.baidu.com/article/9430339, section 4 (rotate, then INT8-quantise).
* Rotated-model explainer -- "量化旋转主模型是什么？一文读懂低比特图像生成模型",
  cloud.baidu.com/article/9432521, section 4 (q = round(R·W / s)).
* INT8 image-text model -- cloud.baidu.com/article/9432337, "how it works"
  (scale per tensor/channel).

OrbitQuant §6.2 (fusing the rotation with the matmul kernels) adds the fused
layer of ``fused.py``: a plain composition of the parts above.

Pin status (what ties each function to something other than itself):

=====================  ===================================================
rng.splitmix64         published SplitMix64 test vector (tests/golden)
rng.rpbh_draw          permutation/sign invariants; no page fixes the RNG
                       (our reading) -- the *choice* is parity-unpinned by
                       the pages, the implementation is pinned
rpbh.hadamard          scipy.linalg.hadamard (library routine) and an
                       independent Kronecker construction
rpbh.rpbh_matrix       literal B·P product at small d; orthogonality;
                       a recursive fast Walsh-Hadamard transform
lloydmax.*             closed form at 1 bit; J. Max (1960) Gaussian tables;
                       centroid condition by independent quadrature;
                       1-D k-means on samples
quant.assign_codes     brute-force nearest level on tiny inputs
quant.pack/unpack      hand-made bit-layout fixture (tests/golden)
quant.quantize_*       invariants (norm, cancellation, INT8 bounds; per-tensor
                       and zero-point variants: range, bound and code-of-0 pins)
qlinear.*              pure-Python triple loop; equal-code closed form
qlinear.int8_levels    J. Max (1960) 16-level table rounded by hand
                       (tests/golden); grid bounds and antisymmetry; the
                       layer within its rounding bound of the exact one
qlinear.e4m3_round     PyTorch's float8_e4m3fn conversion (library routine)
qlinear.fp8_levels     the same Max table rounded to 3 mantissa bits by hand;
                       power-of-two beta; the layer's triple loop, closed
                       form and rounding bound
fused.gelu             y * Phi(y) with Phi from scipy.stats.norm (a library
                       routine); odd-part identity gelu(y) - gelu(-y) = y;
                       published values
fused.qlinear_int8_    composition of pinned parts; a pure-Python triple
  rotate_next          loop and an explicit dense Pi on a tiny case
fused.qlinear_         the same on the code layer: a pure-Python triple
  rotate_next          loop over the levels and an explicit dense Pi
quant.quantize_        steps 2-4 alone: quantize_rotated(Pi x) reproduces
  rotated              quantize_act(x, Pi) exactly; brute-force nearest
                       level on a tiny case
=====================  ===================================================
"""

from .rng import splitmix64, rpbh_draw
from .rpbh import hadamard, rpbh_matrix, rpbh_rows, rpbh_apply
from .lloydmax import lloydmax_unit, lloydmax_table, lloydmax_distortion_unit
from .bf16 import round_to_bf16
from .quant import (assign_codes, pack_codes, unpack_codes, quantize_act, quantize_rotated,
                    quantize_weights_lloydmax, quantize_weights_int8,
                    quantize_weights_int8_asym, rotate_only, EPS)
from .qlinear import (qlinear, qlinear_int8, qlinear_int8_asym, int8_levels, qlinear_int8_levels,
                      e4m3_round, fp8_levels, qlinear_fp8_levels)
from .fused import gelu, qlinear_int8_rotate_next, qlinear_rotate_next

__all__ = [
    "splitmix64", "rpbh_draw", "hadamard", "rpbh_matrix", "rpbh_rows", "rpbh_apply",
    "lloydmax_unit", "lloydmax_table", "lloydmax_distortion_unit",
    "round_to_bf16", "assign_codes", "pack_codes", "unpack_codes",
    "quantize_act", "quantize_rotated", "quantize_weights_lloydmax", "quantize_weights_int8",
    "quantize_weights_int8_asym", "rotate_only", "EPS", "qlinear", "qlinear_int8",
    "qlinear_int8_asym", "int8_levels", "qlinear_int8_levels", "e4m3_round", "fp8_levels",
    "qlinear_fp8_levels", "gelu", "qlinear_int8_rotate_next", "qlinear_rotate_next",
]
