"""CPU float64 oracle (test infrastructure only; see ``oracle/kl.py``)."""
from .kl import (FLAG_IDX_DUP, FLAG_IDX_RANGE, FLAG_NONFINITE, PLAIN, Result, Teacher, Variant,  # noqa: F401
                 bf16_bits_to_f64, effective_mask, kl_loss, kl_loss_from_logits,
                 teacher_distribution)
