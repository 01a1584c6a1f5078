"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module only draws numbers and lays them out.  It holds none of the
decode step's arithmetic: no norm, no rotation, no projection, no selection.
Both the fp64 oracle (``oracle/``) and the CUDA path receive exactly the
arrays produced here, so an oracle input never comes from the CUDA path.

Recipe (Llama-style GQA decoder, bf16 storage):

* projection weights, embedding and LM head: N(0, 0.02) rounded to bf16;
  RMSNorm gains are 1.0;
* KV cache: keys N(0, 1) with four fixed outlier channels scaled by 8, values
  N(0, 1); keys are taken as already rotated (they stand in for the cache a
  dense prefill would have written);
* planted keys (retrieval check): per (layer, kv head) a seeded unit
  direction u; 8 token positions spread evenly over the non-forced pages get
  the key 8 * sqrt(head_dim) * u;
* token ids: seeded uniform integers in [0, vocab);
* observation queries (once-after-prefill selection): per layer, window
  position and query head a vector N(0, 1) in fp32, standing in for the last
  prompt positions' rotated queries;
* batch activations (batched projection): per sequence a N(0, 1) vector
  with a share ``BATCH_SHARED`` of its variance common to the batch, so that
  the sequences' kept channel sets overlap as much as the README's batch
  example assumes.

The weights are drawn layer by layer and kind by kind in a fixed order, the
KV cache chunk by chunk (``KV_CHUNK`` tokens), so that the values depend only
on the seed and the device's generator: a CPU draw and a CUDA draw of the
same seed differ, so every comparison feeds both sides the same draw.
"""
from __future__ import annotations

import math

import torch

# Model shapes.  Field names follow the Hugging Face config fields the ByteCross
# README's byte account reads ("Quick start"); ``page`` is the KV page size.
TINY = dict(n_layers=2, hidden=512, intermediate=1792, n_heads=8, n_kv_heads=2,
            head_dim=64, vocab=4096, rms_eps=1e-5, rope_theta=5e5, page=16)
LLAMA_8B = dict(n_layers=32, hidden=4096, intermediate=14336, n_heads=32,
                n_kv_heads=8, head_dim=128, vocab=128256, rms_eps=1e-5,
                rope_theta=5e5, page=16)

KV_CHUNK = 2048
WEIGHT_STD = 0.02
OUTLIER_SCALE = 8.0


def outlier_channels(head_dim: int) -> list[int]:
    """Four fixed key channels that carry large values (x8)."""
    if head_dim == 128:
        return [7, 31, 70, 115]
    if head_dim == 64:
        return [7, 23, 40, 59]
    return [7 % head_dim, head_dim // 4 + 7, head_dim // 2 + 6, head_dim - 5]


def qkv_width(cfg: dict) -> int:
    return (cfg["n_heads"] + 2 * cfg["n_kv_heads"]) * cfg["head_dim"]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal_bf16(shape, std, g, device) -> torch.Tensor:
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def make_weights(cfg: dict, seed: int = 0, device="cpu") -> dict:
    """Random-init weights of the decoder, in the layouts the library takes.

    Layouts (all bf16, row-major, layers stacked on the leading axis):
      embed   [vocab][hidden]
      lm_head [vocab][hidden]              (output-major, as a Hugging Face lm_head)
      final_norm [hidden], attn_norm/mlp_norm [L][hidden]  (all ones)
      wqkv_t  [L][hidden][(Hq + 2 Hkv) hd] input-channel-major; q columns,
              then k columns, then v columns, head-major inside each block
      wo_t    [L][Hq hd][hidden]
      wgu_t   [L][hidden][2 intermediate]  gate columns first, then up
      wd_t    [L][intermediate][hidden]
    """
    L, d, f = cfg["n_layers"], cfg["hidden"], cfg["intermediate"]
    hq = cfg["n_heads"] * cfg["head_dim"]
    nqkv = qkv_width(cfg)
    V = cfg["vocab"]
    g = _gen(seed, device)
    w = {}
    w["embed"] = _normal_bf16((V, d), WEIGHT_STD, g, device)
    w["lm_head"] = _normal_bf16((V, d), WEIGHT_STD, g, device)
    w["final_norm"] = torch.ones(d, dtype=torch.bfloat16, device=device)
    w["attn_norm"] = torch.ones(L, d, dtype=torch.bfloat16, device=device)
    w["mlp_norm"] = torch.ones(L, d, dtype=torch.bfloat16, device=device)
    for name, shape in (("wqkv_t", (d, nqkv)), ("wo_t", (hq, d)),
                        ("wgu_t", (d, 2 * f)), ("wd_t", (f, d))):
        t = torch.empty((L,) + shape, dtype=torch.bfloat16, device=device)
        for l in range(L):
            t[l] = _normal_bf16(shape, WEIGHT_STD, g, device)
        w[name] = t
    return w


def kv_chunks(cfg: dict, n_tokens: int, seed: int = 1, device="cpu",
              chunk: int = KV_CHUNK):
    """Yield (k, v) bf16 chunks of shape [L][Hkv][c][hd] covering n_tokens.

    Keys are N(0,1) with the outlier channels scaled by 8, values N(0,1).
    """
    L, H, hd = cfg["n_layers"], cfg["n_kv_heads"], cfg["head_dim"]
    g = _gen(seed, device)
    scale = torch.ones(hd, device=device)
    scale[outlier_channels(hd)] = OUTLIER_SCALE
    done = 0
    while done < n_tokens:
        c = min(chunk, n_tokens - done)
        k = torch.randn(L, H, c, hd, generator=g, device=device).mul_(scale)
        v = torch.randn(L, H, c, hd, generator=g, device=device)
        yield k.to(torch.bfloat16), v.to(torch.bfloat16)
        done += c


def make_kv(cfg: dict, n_tokens: int, seed: int = 1, device="cpu"):
    """The whole synthetic cache as two bf16 tensors [L][Hkv][n][hd]."""
    ks, vs = [], []
    for k, v in kv_chunks(cfg, n_tokens, seed, device):
        ks.append(k)
        vs.append(v)
    if not ks:
        shape = (cfg["n_layers"], cfg["n_kv_heads"], 0, cfg["head_dim"])
        e = torch.empty(shape, dtype=torch.bfloat16, device=device)
        return e, e.clone()
    return torch.cat(ks, dim=2), torch.cat(vs, dim=2)


def planted_positions(n_tokens: int, page: int, sinks: int, recent: int,
                      count: int = 8, slot: int = 5) -> list[int]:
    """Token positions of the planted keys: ``count`` pages spread evenly
    over the pages that are neither sinks nor recent, one key per page."""
    P = -(-(n_tokens + 1) // page)          # pages once the next token lands
    lo, hi = sinks, P - recent
    if hi - lo < count:
        raise ValueError("context too short for planted keys")
    pages = [lo + (i * (hi - lo)) // count + (hi - lo) // (2 * count)
             for i in range(count)]
    return [p * page + min(slot, page - 1) for p in pages]


def plant_keys(k: torch.Tensor, positions: list[int], seed: int = 7,
               first_token: int = 0) -> torch.Tensor:
    """Overwrite keys in place: for each (layer, kv head) a seeded unit
    direction u, and key 8*sqrt(hd)*u at every planted position that falls in
    this chunk ``[first_token, first_token + k.shape[2])``."""
    L, H, c, hd = k.shape
    g = _gen(seed, "cpu")
    u = torch.randn(L, H, hd, generator=g, dtype=torch.float64)
    u = u / u.norm(dim=-1, keepdim=True)
    key = (OUTLIER_SCALE * math.sqrt(hd) * u).to(torch.bfloat16).to(k.device)
    for pos in positions:
        if first_token <= pos < first_token + c:
            k[:, :, pos - first_token, :] = key
    return k


def obs_queries(cfg: dict, n_obs: int, seed: int = 11, device="cpu") -> torch.Tensor:
    """Observation-window queries f32 [L][n_obs][Hq][hd], N(0, 1)."""
    g = _gen(seed, device)
    shape = (cfg["n_layers"], n_obs, cfg["n_heads"], cfg["head_dim"])
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


# Share of each batch activation's variance carried by a component common to
# the batch: with it the union of four sequences' top-50% channel sets covers
# about 92% of the channels, the union fraction the ByteCross README's
# crossover_batch example takes for four sequences ("Usage: The byte account").
BATCH_SHARED = 0.37


def batch_activations(batch: int, d: int, shared: float = BATCH_SHARED, seed: int = 13,
                      device="cpu") -> torch.Tensor:
    """Projection inputs of a batch of sequences, f32 [batch][d]:
    sqrt(shared) * z0 + sqrt(1 - shared) * z_b with z0, z_b ~ N(0, 1)."""
    g = _gen(seed, device)
    z0 = torch.randn(1, d, generator=g, device=device, dtype=torch.float32)
    zb = torch.randn(batch, d, generator=g, device=device, dtype=torch.float32)
    return math.sqrt(shared) * z0 + math.sqrt(1.0 - shared) * zb


def tokens(n: int, vocab: int, seed: int = 2) -> list[int]:
    g = _gen(seed, "cpu")
    return torch.randint(0, vocab, (n,), generator=g).tolist()


def bf16_bits(t: torch.Tensor):
    """A bf16 tensor's bit patterns as a host numpy uint16 array."""
    import numpy as np
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
