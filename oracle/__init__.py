"""CPU oracle for multi-scale retention (test infrastructure only; see
retention_oracle.py).  Only tests/, __graft_entry__.smoke() and bench.py's
CPU legs may import it."""
from .retention_oracle import (  # noqa: F401
    backward, chunkwise, decay_mask, gated, group_norm, parallel, recurrent, rel_frobenius, rotate,
    step, swish,
)
