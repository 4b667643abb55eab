"""Host-side set logic of the synthetic decode loop, on CPU tensors: the next
query set Q = T + the front beta_m masks, and the next tracked set."""
import torch

from kv_cache_attention_fdllm_b200 import decode_loop as DL


def test_query_set_front_masks_then_fillers():
    N, beta_m = 20, 4
    decoded = torch.zeros((2, N), dtype=torch.bool)
    decoded[:, :10] = True
    decoded[1, 10:18] = True              # sequence 1 has only 2 masks left (18, 19)
    T = torch.tensor([[2, 5, 9], [1, 3, 4]], dtype=torch.int32)
    q_idx, q_masked, front = DL.query_set(decoded, T, beta_m)
    assert q_idx.dtype == torch.int32 and q_masked.dtype == torch.int8
    assert q_idx[0].tolist() == [2, 5, 9, 10, 11, 12, 13]
    assert q_masked[0].tolist() == [0, 0, 0, 1, 1, 1, 1]
    row = q_idx[1].tolist()
    assert row[:3] == [1, 3, 4] and row[3:5] == [18, 19]
    assert q_masked[1].tolist() == [0, 0, 0, 1, 1, 0, 0]
    # fillers: decoded slots outside T
    assert all(bool(decoded[1, j]) and j not in (1, 3, 4) for j in row[5:])
    for b in range(2):
        assert len(set(q_idx[b].tolist())) == q_idx.shape[1]


def test_next_tracked_keeps_rank_order_of_decoded_slots():
    decoded = torch.zeros((1, 12), dtype=torch.bool)
    decoded[0, [1, 4, 6, 7, 11]] = True
    ranked = torch.tensor([[9, 4, -1, 11, 3, 6, 1, 7]], dtype=torch.int32)
    assert DL.next_tracked(ranked, decoded, 3).tolist() == [[4, 11, 6]]


def test_traffic_model_favours_the_fused_step():
    cfg = DL.LoopConfig(B=8, n_prompt=512, n_gen=512)
    t = DL.algorithmic_bytes_per_layer(cfg, cfg.beta_t + cfg.beta_m)
    assert t["full_recompute"] > t["fused"] > 3 * cfg.H * cfg.dh * cfg.D * 2
