"""B200-native per-round hot path of DSpark-style speculative decoding.

The computation lives in libdspark.so (hand-written CUDA for sm_100a behind
the C ABI of include/dspark.h); this package is its ctypes binding plus a
helper that runs one round (draft -> schedule -> verify) on one stream.
"""
from .binding import (DSPARK_BF16, DSPARK_F32, DSparkError, LIB_PATH, dspark_advance_anchor, dspark_calibrate,
                      dspark_markov_draft, dspark_markov_draft_b, dspark_rnn_draft, dspark_rnn_draft_b,
                      dspark_read_device_error, dspark_schedule, dspark_status_string, dspark_verify,
                      dspark_verify_b, dspark_workspace_bytes, dspark_workspace_init)

__all__ = ["DSPARK_BF16", "DSPARK_F32", "DSparkError", "LIB_PATH", "dspark_advance_anchor", "dspark_calibrate",
           "dspark_markov_draft", "dspark_markov_draft_b", "dspark_rnn_draft", "dspark_rnn_draft_b",
           "dspark_read_device_error", "dspark_schedule", "dspark_status_string", "dspark_verify",
           "dspark_verify_b", "dspark_workspace_bytes", "dspark_workspace_init"]
