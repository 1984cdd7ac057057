"""frnnt: fused RNN-T joint network + transducer loss (forward and backward)
for B200 (sm_100a), behind the C ABI declared in include/frnnt.h.

``rnn_joint_network_02_b200.frnnt`` is the Python binding of libfrnnt.so;
``rnn_joint_network_02_b200.synth`` draws seeded synthetic batches.
"""

from . import frnnt  # noqa: F401
from .frnnt import fwd_bwd, workspace_size  # noqa: F401
