"""fp64 CPU oracle (test infrastructure only; see rnnt_oracle's header)."""
from .rnnt_oracle import (STATUS_BOUNDS, STATUS_LABEL, STATUS_LENGTH, OracleResult, UtteranceLattice,  # noqa: F401
                          alpha_lattice, band_mask, beta_lattice, best_alignment, fwd_bwd, joint_logits, lae,
                          log_sum_exp_last, loss_only, projections, validate,
                          validate_bounds, viterbi_lattice)
from .tdt_oracle import (STATUS_DURATIONS, TdtResult, tdt_alpha, tdt_beta, tdt_edge_posteriors,  # noqa: F401
                         tdt_fwd_bwd, tdt_log_p_from_alpha, tdt_loss_only, validate_durations)
