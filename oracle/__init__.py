"""Float64 CPU oracle (test infrastructure only; see ``spa_oracle``)."""
from .spa_oracle import *  # noqa: F401,F403
from .spa_oracle import (attend, bf16_bits_to_f64, decode, decode_inputs, f64_to_bf16_bits,  # noqa: F401
                         index_append, index_cache_for, index_probs, index_rows, rope,
                         rope_inv_freq, sink_window, softmax, top_k, top_p, block_top_p, BLOCK)
