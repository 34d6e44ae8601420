"""Block-diffusion decoding loop on a small synthetic model.

The method's outer loops ("Fast-dLLM v2: Efficient Block-Diffusion LLM",
overall framework and key designs 3-4): blocks of 32 tokens are decoded
left to right; inside a block, denoising steps run until no position is
[MASK], each step being block attention over [cache ; block] followed by the
confidence-aware unmask; a finished block's K/V are committed to the
block-level cache as read-only context for the blocks after it.

No trained weights are available, so the model is a synthetic single layer
with seeded random weights: x = E[token] (row V of E is the [MASK]
embedding), q/k/v = x Wq / Wk / Wv, h = x + attn(q, k, v) Wo, LM head W.
The embedding and projections are torch glue; attention (with RoPE),
unmask and cache commit are the library's kernels through the C ABI.  A
finished block is run once more with its final tokens to produce the K/V it
commits and the last hidden row the next block's position 0 reads.

With ``dual_cache`` the loop keeps the sub-block DualCache of the current
block (same pages, key design 3; "2.5x inference speedup" article,
"Acceleration engine" item 1; approximate by the notes' own account): at the
first step of each active sub-block the whole block is run and its K, V and
hidden rows are cached; at the following steps of that sub-block only the
active sub-block's rows are fresh, the attention reading the cached K/V of
the other rows and the unmask rule the cached hidden rows outside the active
sub-block.  Only the unmask rule's candidates are scored then
(``bd_confidence_select_active``).  In this one-layer model the saving the
cache brings to a deep model (projections and MLPs of the inactive rows) is
not there to measure; the loop shows the policy and its decisions.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from . import bd
from .workloads import BLOCK, MASK_TOKEN, normal


@dataclasses.dataclass(frozen=True)
class TinyModelConfig:
    vocab: int = 512
    hidden: int = 256
    n_heads_q: int = 4
    n_heads_kv: int = 2
    head_dim: int = 64
    rope_theta: float = 1e4
    w_std: float = 0.5       # LM head scale: logits of std ~8, decisive but not one-hot
    seed: int = 7


class TinyModel:
    """Seeded random weights (fp32, host arrays) of the synthetic layer."""

    def __init__(self, cfg: TinyModelConfig):
        self.cfg = cfg
        V, H, d = cfg.vocab, cfg.hidden, cfg.head_dim
        nq, nkv = cfg.n_heads_q * d, cfg.n_heads_kv * d
        r = lambda tag, shape, std: normal([cfg.seed, tag], shape, std, "f32")
        self.E = r(1, (V + 1, H), 1.0)            # row V: the [MASK] embedding
        self.Wq = r(2, (H, nq), H ** -0.5)
        self.Wk = r(3, (H, nkv), H ** -0.5)
        self.Wv = r(4, (H, nkv), H ** -0.5)
        self.Wo = r(5, (nq, H), nq ** -0.5)
        self.W = r(6, (V, H), cfg.w_std)

    def device(self, device="cuda"):
        return {k: torch.from_numpy(getattr(self, k)).to(device)
                for k in ("E", "Wq", "Wk", "Wv", "Wo", "W")}


def mask_bits(tokens: torch.Tensor) -> torch.Tensor:
    """[B, 32] tokens -> [B] mask words (uint32 bit patterns held as int32),
    bit i set where position i is [MASK]."""
    m = (tokens == MASK_TOKEN).to(torch.int64)
    w = (m << torch.arange(BLOCK, device=tokens.device)).sum(dim=1)
    return torch.where(w >= 2 ** 31, w - 2 ** 32, w).to(torch.int32)


def decode(model: TinyModel, prompt: np.ndarray, n_blocks: int, tau: float, sub_block: int,
           device="cuda", dual_cache: bool = False) -> dict:
    """Decode n_blocks blocks after a prompt of whole blocks, exactly or with
    the sub-block DualCache.

    Returns dict(tokens [B, P + 32 n_blocks], steps [n_blocks, B]: denoising
    steps each sequence needed per block, unmasked [n_blocks][step] list of
    [B] unmask bit words, refreshes: DualCache refresh steps summed over the
    sequences).
    """
    cfg = model.cfg
    B, P = prompt.shape
    assert P % BLOCK == 0 and P > 0
    Hq, Hkv, d, H, V = cfg.n_heads_q, cfg.n_heads_kv, cfg.head_dim, cfg.hidden, cfg.vocab
    w = model.device(device)
    shape = bd.make_shape(Hq, Hkv, d, "f32", cfg.rope_theta)
    cache = bd.KVCache(shape, B, P // BLOCK + n_blocks, device)
    seq_ids = list(range(B))
    out_blk = torch.empty((B, BLOCK, Hq, d), dtype=torch.float32, device=device)
    sel_ws = torch.zeros(bd.bd_confidence_select_workspace_size("f32", B, H, V),
                         dtype=torch.uint8, device=device)
    unmask = torch.zeros(B, dtype=torch.int32, device=device)

    def project(tokens: torch.Tensor):
        x = w["E"][torch.where(tokens == MASK_TOKEN, torch.full_like(tokens, V), tokens).long()]
        q = (x @ w["Wq"]).view(B, BLOCK, Hq, d).contiguous()
        k = (x @ w["Wk"]).view(B, BLOCK, Hkv, d).contiguous()
        v = (x @ w["Wv"]).view(B, BLOCK, Hkv, d).contiguous()
        return x, q, k, v

    def attend(x, q, k, v):
        """Hidden rows of one block over the current cache, given its pre-RoPE k, v."""
        ws = torch.empty(max(bd.bd_block_attn_workspace_size(cache), 256), dtype=torch.uint8,
                         device=device)
        bd.bd_block_attn(cache, q, k.contiguous(), v.contiguous(), out_blk, ws)
        return (x + out_blk.view(B, BLOCK, Hq * d) @ w["Wo"]).contiguous()

    def forward(tokens: torch.Tensor):
        """Hidden rows and pre-RoPE k, v of one block over the current cache."""
        x, q, k, v = project(tokens)
        return attend(x, q, k, v), k, v

    tokens_all = [torch.from_numpy(np.ascontiguousarray(prompt, np.int32)).to(device)]
    h_prev = torch.zeros((B, H), dtype=torch.float32, device=device)
    for b in range(P // BLOCK):  # prefill, block by block
        h, k, v = forward(tokens_all[0][:, b * BLOCK:(b + 1) * BLOCK].contiguous())
        bd.bd_cache_commit(cache, k, v, seq_ids, 1)
        h_prev = h[:, BLOCK - 1].contiguous()
    steps = np.zeros((n_blocks, B), dtype=np.int64)
    unmasked = []
    refreshes = 0
    sub_of = torch.arange(BLOCK, device=device) // sub_block
    for b in range(n_blocks):
        tok = torch.full((B, BLOCK), MASK_TOKEN, dtype=torch.int32, device=device)
        log = []
        cached_sub = torch.full((B,), -1, dtype=torch.long, device=device)
        Kc = torch.zeros((B, BLOCK, Hkv, d), dtype=torch.float32, device=device)
        Vc = torch.zeros_like(Kc)
        Hc = torch.zeros((B, BLOCK, H), dtype=torch.float32, device=device)
        for _ in range(BLOCK + 1):  # at least one token per sequence and step: <= 32 steps
            bits = mask_bits(tok)
            if not bool((tok == MASK_TOKEN).any()):
                break
            still = (tok == MASK_TOKEN).any(dim=1).cpu().numpy()
            steps[b] += still
            if dual_cache:
                x, q, k, v = project(tok)
                # active sub-block: the one holding the first masked position
                a = (tok == MASK_TOKEN).to(torch.int32).argmax(dim=1).long() // sub_block
                rows = sub_of[None, :] == a[:, None]                      # [B, 32]
                refresh = cached_sub != a
                refreshes += int(refresh[torch.from_numpy(still).to(device)].sum())
                Kc = torch.where(refresh[:, None, None, None], k, Kc)
                Vc = torch.where(refresh[:, None, None, None], v, Vc)
                cached_sub = torch.where(refresh, a, cached_sub)
                h_new = attend(x, q, torch.where(rows[:, :, None, None], k, Kc),
                               torch.where(rows[:, :, None, None], v, Vc))
                Hc = torch.where(refresh[:, None, None], h_new, Hc)
                h = torch.where(rows[:, :, None], h_new, Hc).contiguous()
                bd.bd_confidence_select_active("f32", B, H, V, h, h_prev, w["W"], bits, tau,
                                               sub_block, tok, unmask, None, None, sel_ws)
            else:
                h, _, _ = forward(tok)
                bd.bd_confidence_select("f32", B, H, V, h, h_prev, w["W"], bits, tau, sub_block,
                                        tok, unmask, None, None, sel_ws)
            log.append(unmask.cpu().numpy().view(np.uint32).copy())
        h, k, v = forward(tok)       # the finished block with its final tokens
        bd.bd_cache_commit(cache, k, v, seq_ids, 1)
        h_prev = h[:, BLOCK - 1].contiguous()
        tokens_all.append(tok)
        unmasked.append(log)
    return dict(tokens=torch.cat(tokens_all, dim=1).cpu().numpy(), steps=steps, unmasked=unmasked,
                refreshes=refreshes)


def main():
    """Run the loop on the synthetic model and print one JSON line: tokens
    decoded per second (wall clock, host glue included) and steps per block."""
    import argparse
    import json
    import time
    ap = argparse.ArgumentParser()
    ap.add_argument("--batch", type=int, default=4)
    ap.add_argument("--prompt-blocks", type=int, default=2)
    ap.add_argument("--blocks", type=int, default=4)
    ap.add_argument("--tau", type=float, default=0.9)
    ap.add_argument("--sub-block", type=int, default=8)
    ap.add_argument("--dual-cache", action="store_true")
    args = ap.parse_args()
    model = TinyModel(TinyModelConfig())
    rng = np.random.default_rng(0)
    prompt = rng.integers(0, model.cfg.vocab, size=(args.batch, BLOCK * args.prompt_blocks))
    decode(model, prompt.astype(np.int32), 1, args.tau, args.sub_block,
           dual_cache=args.dual_cache)  # warm-up
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    r = decode(model, prompt.astype(np.int32), args.blocks, args.tau, args.sub_block,
               dual_cache=args.dual_cache)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    print(json.dumps({"tokens_per_s": args.batch * args.blocks * BLOCK / dt,
                      "mean_steps_per_block": float(r["steps"].mean()),
                      "tau": args.tau, "sub_block": args.sub_block, "batch": args.batch,
                      "dual_cache": args.dual_cache, "refresh_steps": r["refreshes"],
                      "model": dataclasses.asdict(model.cfg)}))


if __name__ == "__main__":
    main()
