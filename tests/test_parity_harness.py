"""The parity harness on the CPU: the oracle run over token shards in spawned
processes gives exactly what one call over all tokens gives (tokens are
independent in the layer), so the full-size GPU comparisons that use it check
every token against the unchanged oracle."""
import numpy as np

import oracle
from ternary_weight_moe_forward_b200 import synth

from parity import oracle_shards


def test_sharded_oracle_equals_one_call():
    shape = synth.CONFIGS["tiny"]["shape"]
    x = synth.activations(70, shape.d_model, seed=2)
    whole = oracle.Layer(shape, synth.layer_weights(shape, seed=0, zipf=1.1)).forward_tokens(x)
    seen = np.zeros(70, bool)
    for tokens, ref in oracle_shards(shape, 0, 1.1, x, shard=16, workers=3):
        assert not seen[tokens].any()
        seen[tokens] = True
        for k, v in ref.items():
            assert np.array_equal(v.view(np.uint8), whole[k][tokens].view(np.uint8)), k
    assert seen.all()
