"""fp64 CPU oracle for the Muon / Dimuon step (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
import this package.  It shares no code with the CUDA library.
"""
from .dimuon_oracle import (  # noqa: F401
    COND_EPS, MOONSHOT_COEF, NS_A, NS_B, NS_C, NS_STEPS, SCALE_BERNSTEIN, SCALE_JORDAN,
    SCALE_MOONSHOT, SCALE_NONE, HParams, StepResult, conditioning, dimuon_step, energies,
    f32, frobenius_normalise, momentum_update, muon_step, newton_schulz,
    optimizer_step, polar_factor_svd, round_bf16, scale_factor, store_round,
    top_column_share, vector_matrix_shape, vector_step, vector_to_matrix, matrix_to_vector,
)
