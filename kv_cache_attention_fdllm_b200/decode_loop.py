"""A multi-step synthetic decode loop over the library's calls.

Flash-dLLM review, "How It Works": every denoising step runs the draft pass
(Step 1: Draft, the fused KV-cache step over Q = T + the front beta_m masks), the
epsilon split of the masked rows, a Flash-Verify pass over the exploratory rows
with the gamma prefix acceptance (Step 1: Verification), and the choice of the
next tracked set (Step 1: Cache selection).  This driver repeats that over L
random-weight layers until every generated position is decoded, to measure
steps/s and what the fused step moves against a full recompute.

There is no model and no data: weights, hidden states, caches and the logits that
stand in for the LM head are seeded random tensors (the logits get one spike per
row so that confidences spread over 0.3-0.99).  Between layers the attention
output of the rows in Q is added to their hidden state, a stand-in for the rest
of the transformer block, so each layer's step reads what the previous one
wrote.  Every step of the method itself runs in the library's kernels.

Policies the pages leave to the caller (stated here, used below):
  * when neither the epsilon split nor the verification commits a row, the
    most confident masked row is committed, so that every step makes progress;
  * T_v of the verify pass is the current tracked set;
  * the exploratory set S of a step has the same size in every sequence (the
    smallest count over the batch), in decoding order (confidence descending);
  * the tracked set is chosen from the middle layer's attention.  The slots
    resolved in the step take part in the ranking, as on the page: the middle
    layer ranks the decoded slots and the step's masked positions, and T becomes the first beta_t of that ranking that are decoded
    once the step has committed its rows.
"""
from __future__ import annotations

import argparse
import json
import math
import time
from dataclasses import asdict, dataclass

import torch

from . import api as F


@dataclass
class LoopConfig:
    B: int = 1
    n_prompt: int = 512
    n_gen: int = 256
    H: int = 32
    dh: int = 128
    L: int = 4
    beta_m: int = 64
    beta_t: int = 80
    eps: float = 0.9
    gamma: float = 0.8
    vocab: int = 32000
    seed: int = 7
    max_steps: int = 10000
    causal_cross: bool = False

    @property
    def N(self) -> int:
        return self.n_prompt + self.n_gen

    @property
    def D(self) -> int:
        return self.H * self.dh


def _synthetic_logits(gen, B, R, V, device, spike_tok=None):
    """N(0,1) logits with one spike per row giving a confidence u ~ U(0.3, 0.99)."""
    z = torch.randn((B, R, V), generator=gen, device=device)
    u = 0.3 + 0.69 * torch.rand((B, R), generator=gen, device=device)
    spike = math.log(V) + 0.5 + torch.log(u / (1 - u))
    tok = spike_tok if spike_tok is not None else torch.randint(0, V, (B, R), generator=gen, device=device)
    z.scatter_(2, tok.long().unsqueeze(-1), spike.unsqueeze(-1))
    return z.contiguous(), tok.int()


def algorithmic_bytes_per_layer(cfg: LoopConfig, nq: int) -> dict:
    """Bytes one layer's draft pass must move, against recomputing every row
    (the same projection and attention over all N positions, no cache)."""
    e, E, D, N, B = 2, cfg.H * cfg.dh, cfg.D, cfg.N, cfg.B
    w = 3 * E * D * e
    fused = w + B * nq * D * e + 2 * B * N * E * e + 3 * B * nq * E * e + B * nq * E * e
    full = w + B * N * D * e + 2 * B * N * E * e * 2 + B * N * E * e * 2
    return {"fused": fused, "full_recompute": full}


def query_set(decoded, T, beta_m):
    """Q of the next step: the tracked set T, then the front beta_m masked
    positions in position order.  When fewer masks remain, decoded slots that
    are not in T fill the rest, flagged as non-masked rows.

    decoded bool [B, N], T int32 [B, beta_t].  Returns (q_idx int32 [B, beta_t +
    beta_m], q_masked int8 [B, beta_t + beta_m], front int64 [B, beta_m])."""
    B, N = decoded.shape
    dev = decoded.device
    ar = torch.arange(N, device=dev)
    masks_left = (~decoded).sum(dim=1)
    key = torch.where(decoded, N + ar, ar)               # masks first, in position order
    front = torch.argsort(key.float(), dim=1)[:, :beta_m]
    m_cnt = torch.clamp(masks_left, max=beta_m)
    is_T = torch.zeros((B, N), dtype=torch.bool, device=dev)
    is_T.scatter_(1, T.long(), True)
    fill = torch.argsort((is_T | ~decoded).float() * 2 + (ar.float() / N), dim=1)  # decoded, non-T
    slot_j = torch.arange(beta_m, device=dev).unsqueeze(0)
    front = torch.where(slot_j < m_cnt.unsqueeze(1), front, fill[:, :beta_m])
    q_idx = torch.cat([T.int(), front.int()], dim=1).contiguous()
    q_masked = torch.cat([torch.zeros((B, T.shape[1]), dtype=torch.int8, device=dev),
                          (slot_j < m_cnt.unsqueeze(1)).to(torch.int8)], dim=1).contiguous()
    return q_idx, q_masked, front


def next_tracked(ranked, decoded, beta_t):
    """The next tracked set: the first beta_t slots of the ranking (-1 entries
    skipped) that are decoded once the step has committed its rows, in rank
    order.  ranked int32 [B, K], decoded bool [B, N]."""
    ok = (ranked >= 0) & torch.gather(decoded, 1, ranked.clamp(min=0).long())
    first = torch.argsort((~ok).to(torch.int8), dim=1, stable=True)[:, :beta_t]
    return torch.gather(ranked, 1, first).contiguous()


def _cpu(t):
    return t.detach().to("cpu", copy=True)


def run(cfg: LoopConfig, device="cuda", trace: dict | None = None) -> dict:
    """Decodes the generated block.  With a dict as `trace`, the first step's
    calls record their inputs and results in it (CPU copies): the draft pass of
    layer 0 and of the middle layer ("draft"), the tracked-set selection
    ("track"), the epsilon split ("split"), the verify pass of layer 0
    ("verify"), the gamma acceptance ("gamma") and the sets the step ends with
    ("sets"), so that each call can be replayed on the same inputs."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed)
    bf = torch.bfloat16
    B, N, D, H, dh = cfg.B, cfg.N, cfg.D, cfg.H, cfg.dh
    nq = cfg.beta_t + cfg.beta_m
    if cfg.beta_t > cfg.n_prompt or cfg.beta_m > cfg.n_gen:
        raise ValueError("beta_t must fit in the prompt and beta_m in the generated block")

    W = [(torch.randn((3 * H * dh, D), generator=gen, device=dev) / math.sqrt(D)).to(bf)
         for _ in range(cfg.L)]
    K = [torch.randn((B, H, N, dh), generator=gen, device=dev).to(bf) for _ in range(cfg.L)]
    V = [torch.randn((B, H, N, dh), generator=gen, device=dev).to(bf) for _ in range(cfg.L)]
    x0 = torch.randn((B, N, D), generator=gen, device=dev).to(bf)
    S_cap = cfg.beta_m
    KS = [torch.zeros((B, H, S_cap, dh), dtype=bf, device=dev) for _ in range(cfg.L)]
    VS = [torch.zeros((B, H, S_cap, dh), dtype=bf, device=dev) for _ in range(cfg.L)]

    ws = F.alloc_workspace(F.fdllm_fused_step_workspace_bytes(B, N, D, H, dh, nq, bf), dev)
    R_max = cfg.beta_t + 2 * S_cap
    ws_v = F.alloc_workspace(F.fdllm_verify_step_workspace_bytes(B, N, D, H, dh, R_max, S_cap, bf), dev)
    ws_a = F.alloc_workspace(F.fdllm_accept_workspace_bytes(B, R_max, cfg.vocab), dev)
    out = torch.empty((B, nq, H * dh), dtype=bf, device=dev)
    track = torch.empty((B, cfg.beta_t + cfg.beta_m), dtype=torch.int32, device=dev)

    decoded = torch.zeros((B, N), dtype=torch.bool, device=dev)
    decoded[:, : cfg.n_prompt] = True
    T = torch.arange(cfg.n_prompt - cfg.beta_t, cfg.n_prompt, device=dev, dtype=torch.int32)
    T = T.unsqueeze(0).expand(B, -1).contiguous()

    steps, committed_total = 0, 0
    per_step_ms, per_step_commit = [], []
    launches0 = F.lib().fdllm_launch_count()
    t_wall = time.perf_counter()
    while steps < cfg.max_steps:
        masks_left = (~decoded).sum(dim=1)
        if int(masks_left.max()) == 0:
            break  # a finished sequence rides along with an all-decoded Q until then
        rec = trace if (trace is not None and steps == 0) else None
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        q_idx, q_masked, front = query_set(decoded, T, cfg.beta_m)
        if rec is not None:
            rec.update(draft={}, decoded_before=_cpu(decoded), T=_cpu(T), q_idx=_cpu(q_idx),
                       q_masked=_cpu(q_masked), front=_cpu(front), W=[_cpu(w) for w in W])

        # draft pass over the layers; the tracked set comes from the middle layer
        x = x0.clone()
        rows = q_idx.long()
        bidx = torch.arange(B, device=dev).unsqueeze(1)
        for l in range(cfg.L):
            keep = rec is not None and l in (0, cfg.L // 2)
            if keep:
                rec["draft"][l] = {"x": _cpu(x), "k_in": _cpu(K[l]), "v_in": _cpu(V[l])}
            F.fdllm_fused_step(x, q_idx, W[l], K[l], V[l], out, ws)
            if keep:
                rec["draft"][l].update(out=_cpu(out), k_out=_cpu(K[l]), v_out=_cpu(V[l]))
            if l == cfg.L // 2:
                cand = decoded.clone()
                cand.scatter_(1, front.long(), q_masked[:, cfg.beta_t:].bool() | torch.gather(cand, 1, front.long()))
                cand8 = cand.to(torch.int8).contiguous()
                mass = torch.empty((B, N), dtype=torch.float32, device=dev) if rec is not None else None
                F.fdllm_track_select(q_masked, cand8, K[l], track, ws, mass=mass)
                if rec is not None:
                    rec["track"] = {"layer": l, "candidate": _cpu(cand8), "track": _cpu(track),
                                    "mass": _cpu(mass)}
            x[bidx, rows] = x[bidx, rows] + out
        # epsilon split of the masked rows (stand-in LM head: synthetic logits)
        R1 = cfg.beta_m
        logits, draft_tok = _synthetic_logits(gen, B, R1, cfg.vocab, dev)
        kind = torch.ones((B, R1), dtype=torch.int8, device=dev)
        top1 = torch.empty((B, R1), dtype=torch.int32, device=dev)
        conf = torch.empty((B, R1), dtype=torch.float32, device=dev)
        flags = torch.empty((B, R1), dtype=torch.uint8, device=dev)
        n_acc = torch.empty((B,), dtype=torch.int32, device=dev)
        F.fdllm_accept(logits, kind, None, None, top1, conf, flags, n_acc, ws_a, eps=cfg.eps,
                       gamma=cfg.gamma)
        if rec is not None:
            rec["split"] = {"logits": _cpu(logits), "kind": _cpu(kind), "top1": _cpu(top1),
                            "conf": _cpu(conf), "flags": _cpu(flags)}
        valid = q_masked[:, cfg.beta_t:].bool()
        commit = ((flags & F.FLAG_COMMIT) != 0) & valid
        # exploratory rows in decoding order (confidence descending)
        explore = valid & ~commit
        n_s = int(explore.sum(dim=1).min())
        n_s = min(n_s, S_cap)
        newly = torch.zeros((B, N), dtype=torch.bool, device=dev)
        newly.scatter_(1, front.long(), commit)
        if n_s > 0:
            c_ord = torch.where(explore, conf, torch.full_like(conf, -1.0))
            pick = torch.argsort(-c_ord, dim=1)[:, :n_s]     # rows of the masked block
            s_pos = torch.gather(front, 1, pick)
            R = cfg.beta_t + 2 * n_s
            pos = torch.cat([T, s_pos.int(), s_pos.int()], dim=1).contiguous()
            view = torch.cat([torch.zeros((B, cfg.beta_t), dtype=torch.int8, device=dev),
                              torch.ones((B, n_s), dtype=torch.int8, device=dev),
                              torch.full((B, n_s), 2, dtype=torch.int8, device=dev)], 1).contiguous()
            rank = torch.cat([torch.zeros((B, cfg.beta_t), dtype=torch.int32, device=dev),
                              torch.arange(n_s, dtype=torch.int32, device=dev).expand(B, -1),
                              torch.arange(n_s, dtype=torch.int32, device=dev).expand(B, -1)],
                             1).contiguous()
            xv = x0.clone()
            rv = pos.long()
            out_v = torch.empty((B, R, H * dh), dtype=bf, device=dev)
            for l in range(cfg.L):
                x_rows = xv[bidx, rv].contiguous()
                if rec is not None and l == 0:
                    rec["verify"] = {"x_rows": _cpu(x_rows), "pos": _cpu(pos), "view": _cpu(view),
                                     "rank": _cpu(rank), "k_in": _cpu(K[l]), "v_in": _cpu(V[l]),
                                     "ks_in": _cpu(KS[l]), "vs_in": _cpu(VS[l])}
                # the first n_s side slots take the mask view; the rest stay unused
                F.fdllm_verify_step(x_rows, pos, view, rank, W[l], K[l], V[l], KS[l], VS[l], out_v,
                                    ws_v, causal_cross=cfg.causal_cross)
                if rec is not None and l == 0:
                    rec["verify"].update(out=_cpu(out_v), k_out=_cpu(K[l]), v_out=_cpu(V[l]),
                                         ks_out=_cpu(KS[l]), vs_out=_cpu(VS[l]))
                xv[bidx, rv] = xv[bidx, rv] + out_v
            # mask-view predictions agree with the draft with probability 0.8
            d_tok = torch.gather(draft_tok, 1, pick)
            agree = torch.rand((B, n_s), generator=gen, device=dev) < 0.8
            m_tok = torch.where(agree, d_tok, (d_tok + 1) % cfg.vocab)
            lg_v, _ = _synthetic_logits(gen, B, n_s, cfg.vocab, dev, spike_tok=m_tok)
            kind_v = torch.full((B, n_s), 2, dtype=torch.int8, device=dev)
            rank_v = torch.arange(n_s, dtype=torch.int32, device=dev).expand(B, -1).contiguous()
            t1 = torch.empty((B, n_s), dtype=torch.int32, device=dev)
            c1 = torch.empty((B, n_s), dtype=torch.float32, device=dev)
            f1 = torch.empty((B, n_s), dtype=torch.uint8, device=dev)
            F.fdllm_accept(lg_v, kind_v, d_tok.contiguous(), rank_v, t1, c1, f1, n_acc, ws_a,
                           eps=cfg.eps, gamma=cfg.gamma)
            acc_v = (f1 & F.FLAG_ACCEPT) != 0
            if rec is not None:
                rec["gamma"] = {"logits": _cpu(lg_v), "kind": _cpu(kind_v), "ref_tok": _cpu(d_tok),
                                "rank": _cpu(rank_v), "top1": _cpu(t1), "conf": _cpu(c1),
                                "flags": _cpu(f1), "n_accept": _cpu(n_acc), "s_pos": _cpu(s_pos)}
            newly.scatter_(1, s_pos.long(), acc_v | torch.gather(newly, 1, s_pos.long()))
        # progress policy: at least the most confident masked row per sequence
        none = ~newly.any(dim=1)
        if bool(none.any()):
            best = torch.argmax(torch.where(valid, conf, torch.full_like(conf, -1.0)), dim=1)
            bpos = torch.gather(front, 1, best.unsqueeze(1)).squeeze(1)
            newly[none, bpos[none]] = True
        newly &= ~decoded
        decoded |= newly
        T = next_tracked(track, decoded, cfg.beta_t)
        if rec is not None:
            rec["sets"] = {"newly": _cpu(newly), "progress_forced": _cpu(none),
                           "decoded": _cpu(decoded), "T_next": _cpu(T), "n_s": n_s}
        ev1.record()
        torch.cuda.synchronize()
        for w in (ws, ws_v, ws_a):
            if F.fdllm_get_status(w) != F.OK:
                raise RuntimeError("device status set during the decode loop")
        per_step_ms.append(ev0.elapsed_time(ev1))
        per_step_commit.append(int(newly.sum()))
        committed_total += per_step_commit[-1]
        steps += 1
    wall = time.perf_counter() - t_wall
    traffic = algorithmic_bytes_per_layer(cfg, nq)
    gpu_ms = sum(per_step_ms)
    return {
        "config": asdict(cfg),
        "steps": steps,
        "all_decoded": bool(decoded.all()),
        "tokens_decoded": committed_total,
        "tokens_per_step": committed_total / max(1, steps) / B,
        "steps_per_s": steps / (gpu_ms / 1e3) if gpu_ms else None,
        "ms_per_step": gpu_ms / max(1, steps),
        "wall_s": wall,
        "kernel_launches": int(F.lib().fdllm_launch_count() - launches0),
        "draft_bytes_per_layer": traffic["fused"],
        "full_recompute_bytes_per_layer": traffic["full_recompute"],
        "draft_traffic_saving": traffic["full_recompute"] / traffic["fused"],
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    for f, v in asdict(LoopConfig()).items():
        ap.add_argument("--" + f.replace("_", "-"), type=type(v) if not isinstance(v, bool) else int,
                        default=v)
    a = ap.parse_args()
    cfg = LoopConfig(**{f: (bool(getattr(a, f)) if isinstance(v, bool) else getattr(a, f))
                        for f, v in asdict(LoopConfig()).items()})
    print(json.dumps(run(cfg)))


if __name__ == "__main__":
    main()
