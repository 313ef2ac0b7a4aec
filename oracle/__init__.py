"""fp64 CPU oracle (test infrastructure; never on the product path)."""

from .eqlin_oracle import (  # noqa: F401
    D8_COORDS,
    cyclic_backward_data,
    cyclic_counts,
    cyclic_dense_matrix,
    cyclic_forward,
    cyclic_weight_grad,
    d8_chars_1d,
    d8_counts,
    d8_dense_operator,
    d8_elements,
    d8_forward,
    d8_inv,
    d8_mul,
    d8_Q,
    d8_regular_perm,
    d8_rho_E,
    d8_slot,
    gelu_exact,
    negacyclic_forward,
    rel_frobenius,
)
