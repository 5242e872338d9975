"""KDA (Kimi Delta Attention) on B200: chunked prefill and decode through the
C ABI of libkda.so (include/kda.h).  Importing the package does not load the
library; the first call does, and fails loudly if it is missing."""
from .binding import (BETA_LOGIT, GATE_CHANNEL, GATE_FUSED, GATE_NONE, GATE_SCALAR, KDA_BF16,
                      KDA_F32, NORM_K, NORM_Q, KDAError, kda_chunk_bwd, kda_chunk_fwd, kda_chunk_fwd_ex,
                      kda_decode_ex, kda_decode_step, kda_device_status,
                      kda_selftest_wait_timeout, kda_status_string, load_library)

__all__ = ["BETA_LOGIT", "GATE_CHANNEL", "GATE_FUSED", "GATE_NONE", "GATE_SCALAR", "KDA_BF16",
           "KDA_F32", "NORM_K", "NORM_Q", "KDAError", "kda_chunk_bwd", "kda_chunk_fwd", "kda_chunk_fwd_ex",
           "kda_decode_ex", "kda_decode_step", "kda_device_status", "kda_selftest_wait_timeout",
           "kda_status_string", "load_library"]
