"""CPU oracle (test infrastructure only; see switch_oracle's header)."""
from .switch_oracle import (capacity, router, dispatch, expert, expert_ffn,  # noqa: F401
                            combine, aux_loss, layer_forward, token_outputs)
