"""The precision reading of the 16-bit path, measured on the CPU.

The pages compute the forward pass in bf16. For the 8B shapes (32 layers,
seeded N(0, 0.02) weights) this replays the GPU path's rounding points
(tests/precision_emulation.py) with bf16 and with fp16 roundings and compares
the last-token logits with the exact computation (float64, no rounding):
bf16 roundings alone put the logits beyond the 2e-2 relative-L2 bound of the
16-bit configurations, fp16 roundings (three more mantissa bits, same tensor
rate) keep them well inside it. This is why the library's default 16-bit
policy keeps bf16 weight values but rounds activations to fp16.
"""
import numpy as np
import pytest

import seeded_inputs as si
from oracle import Params
from tests.helpers import rel_l2
from tests.precision_emulation import last_token_logits, no_round, round_bf16, round_fp16


@pytest.mark.slow
def test_bf16_activations_exceed_the_bound_fp16_stay_inside():
    p = Params(4096, 32, 32, 8, 128256, 14336)
    toks = si.tokens(1, 48, p.vocab_size)
    res = last_token_logits(0, p, toks, {'exact': (no_round, np.float64),
                                          'bf16': (round_bf16, np.float32),
                                          'fp16': (round_fp16, np.float32)})
    e_bf16 = rel_l2(res['bf16'], res['exact'])
    e_fp16 = rel_l2(res['fp16'], res['exact'])
    print(f'32-layer 8B logits, relative L2 from exact: bf16 roundings {e_bf16:.3e}, fp16 roundings {e_fp16:.3e}')
    assert e_bf16 > 2e-2
    assert e_fp16 < 1e-2
    assert e_bf16 > 4 * e_fp16
