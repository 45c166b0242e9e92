"""CPU oracle of the Hadamard-rotated quantized linear layer (test infrastructure only).

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may
import this package; the product path never does.
"""
from .qs_oracle import *  # noqa: F401,F403
from .qs_oracle import QMAX, HADAMARD_BLOCK, WEIGHT_SCALE_FOLD  # noqa: F401
from .gbs_oracle import (  # noqa: F401
    GBS_HIGH_BITS, GBS_LOW_BITS, GbsState, gbs_run, gbs_schedule, gbs_update, l1_distance, l1_terms,
)
from .bgr_oracle import (  # noqa: F401
    BGR_DEFAULT_CANDIDATES, BGR_DEFAULT_ITERATIONS, asym_accumulators, bgr_row, bound_search,
    code_rowsums, grid_codes, grid_error, grid_from_bounds, least_squares_grid, pack_weights_bgr,
    qlinear_bgr, seq_sum,
)
from .sd4_oracle import (  # noqa: F401
    SD4_BLOCK, SD4_DIALECTS, decompose_rows, formatbook, linear_sd4, linear_sd4_decomp,
    lut_tables, pack_codes, pack_decomp, pack_meta, quantize_values,
)
