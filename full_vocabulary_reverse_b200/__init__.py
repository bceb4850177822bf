"""B200-native exact full-vocabulary reverse-KL distillation loss.

The compute runs in ``librkl.so`` (hand-written sm_100a CUDA kernels behind a
C ABI, see ``include/rkl.h``); this package only loads it and marshals
arguments.  There is no CPU or PyTorch fallback: if the library is missing,
every call raises.
"""

from .binding import (  # noqa: F401
    RKLError, lib, compact_rows, forward_hidden, forward_logits, backward,
    forward_logits_pair, backward_logits_pair, forward_with_stats,
    workspace_size, device_error, reverse_kl_hidden, reverse_kl_logits, reverse_kl_logits_pair,
    forward_topk_pair, backward_topk_pair, topk_estimator_logits_pair,
    forward_topk_hidden, backward_topk_hidden, topk_estimator_hidden,
    compact_rows_multi, forward_hidden_multi, backward_hidden_multi, workspace_size_multi, reverse_kl_hidden_multi,
    REDUCE_NONE, REDUCE_TOKEN_MEAN, REDUCE_SEQ_MEAN_NESTED,
    PAYLOAD_HIDDEN, PAYLOAD_LOGITS, PAYLOAD_LOGITS_PAIR,
)
