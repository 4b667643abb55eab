"""The synthetic multi-step decode loop runs every call of the path in sequence
(draft pass per layer, epsilon split, verify pass, gamma acceptance, tracked-set
selection) until the generated block is decoded."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
def test_decode_loop_decodes_everything(causal):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from kv_cache_attention_fdllm_b200 import decode_loop as DL
    cfg = DL.LoopConfig(B=2, n_prompt=32, n_gen=24, H=2, dh=64, L=2, beta_m=8, beta_t=4,
                        vocab=64, seed=3, max_steps=100, causal_cross=causal)
    r = DL.run(cfg)
    assert r["all_decoded"]
    assert r["tokens_decoded"] == cfg.B * cfg.n_gen
    assert 1 <= r["steps"] <= cfg.n_gen
    assert r["kernel_launches"] > 0
    assert r["draft_traffic_saving"] > 1.0
