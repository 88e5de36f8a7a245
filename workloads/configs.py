"""The six synthetic MLA workloads, with their shapes, seeds and input recipes.

Shapes follow DeepSeek-V2/V3 layers: latent width d_c = 512 (kv_lora_rank), decoupled
RoPE key width d_hR = 64 (qk_rope_head_dim), 128 heads of 128 content dims.  No
dataset or trained weight is involved; every tensor is drawn from `workloads.rng` with a
fixed seed per workload and a fixed id per tensor, so both sides of a parity test get
identical bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, Optional, Tuple

import numpy as np
import torch

from . import rng

# one stream id per tensor name, shared by every workload
TENSOR_IDS = {
    "W_DKV": 1, "W_KR": 2, "W_Q": 3, "W_UK": 4, "W_UV": 5, "W_O": 6,
    "h_hist": 7, "h_new": 8, "cache": 9, "q_nope": 10, "q_rope": 11, "lengths": 12, "h": 13,
}


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "decode_layer" | "decode_attn" | "decode_fp8" | "decode_multi" | "prefill"
    B: int
    H: int
    d_model: int              # 0 when the workload starts from given queries
    d_c: int
    d_hR: int
    qk_nope: int
    v_head: int
    dtype: str                # storage type: "f32" or "bf16"; accumulation is always fp32
    seed: int
    ctx: int = 0              # uniform cached length (decode) or sequence length (prefill)
    ctx_range: Optional[Tuple[int, int]] = None   # ragged cached lengths, inclusive
    history: str = ""         # decode_layer: "hidden" (cache built by appending) | "synthetic"
    rope_theta: float = 10000.0
    cache_std: float = 0.5    # synthetic cache rows ~ cache_std * N(0, 1)
    q_len: int = 1            # decode_multi: new tokens per sequence (appended after the ctx rows)
    fold: bool = False        # decode_layer: weights with W_UK folded into W_Q and W_UV into W_O

    @property
    def row(self) -> int:
        """Cache elements per token per layer: the latent plus the decoupled RoPE key."""
        return self.d_c + self.d_hR

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.qk_nope + self.d_hR)


def _seed(n: int) -> int:
    return 0x4D4C41 + n


WORKLOADS: Dict[str, Workload] = {
    # tiny single-layer decode, fp32 end to end; the cache is built by appending 128 tokens
    "tiny_fp32_layer": Workload("tiny_fp32_layer", "decode_layer", B=2, H=4, d_model=256, d_c=64,
                                d_hR=16, qk_nope=32, v_head=32, dtype="f32", seed=_seed(1),
                                ctx=128, history="hidden"),
    # DeepSeek-V3-shaped absorbed decode attention over a uniform 4096-token latent cache
    "v3_decode_b32_ctx4096": Workload("v3_decode_b32_ctx4096", "decode_attn", B=32, H=128, d_model=0,
                                      d_c=512, d_hR=64, qk_nope=128, v_head=128, dtype="bf16",
                                      seed=_seed(2), ctx=4096),
    # ragged long-context decode: 64 sequences with lengths ~ U[1024, 32768]
    "v3_ragged_b64": Workload("v3_ragged_b64", "decode_attn", B=64, H=128, d_model=0, d_c=512,
                              d_hR=64, qk_nope=128, v_head=128, dtype="bf16", seed=_seed(3),
                              ctx_range=(1024, 32768)),
    # full decode layer at V3 sizes: append, query projection, absorbed attention, W_UV, W_O
    "v3_layer_b128_ctx8192": Workload("v3_layer_b128_ctx8192", "decode_layer", B=128, H=128,
                                      d_model=7168, d_c=512, d_hR=64, qk_nope=128, v_head=128,
                                      dtype="bf16", seed=_seed(4), ctx=8192, history="synthetic"),
    # the same layer (same inputs) on folded weights: q_lat = (W_UK^T W_Q) h, out = (W_O W_UV) o_lat
    "v3_layer_folded_b128_ctx8192": Workload("v3_layer_folded_b128_ctx8192", "decode_layer", B=128, H=128,
                                             d_model=7168, d_c=512, d_hR=64, qk_nope=128, v_head=128,
                                             dtype="bf16", seed=_seed(4), ctx=8192, history="synthetic",
                                             fold=True),
    # causal prefill at V2 sizes with materialised K/V
    "v2_prefill_b4_s4096": Workload("v2_prefill_b4_s4096", "prefill", B=4, H=128, d_model=5120,
                                    d_c=512, d_hR=64, qk_nope=128, v_head=128, dtype="bf16",
                                    seed=_seed(5), ctx=4096),
    # the V3 decode workload over an FP8 latent cache (its bf16 rows quantised once, before
    # the step: E4M3 codes with one fp32 scale per token, bf16 rotary key)
    "v3_decode_fp8_b32_ctx4096": Workload("v3_decode_fp8_b32_ctx4096", "decode_fp8", B=32, H=128, d_model=0,
                                          d_c=512, d_hR=64, qk_nope=128, v_head=128, dtype="bf16",
                                          seed=_seed(2), ctx=4096),
    # multi-token decode (speculative verification): 2 new tokens per sequence over 4096
    # cached tokens, paged cache
    "v3_mtp_b32_ctx4096_q2": Workload("v3_mtp_b32_ctx4096_q2", "decode_multi", B=32, H=128, d_model=0,
                                      d_c=512, d_hR=64, qk_nope=128, v_head=128, dtype="bf16",
                                      seed=_seed(6), ctx=4096, q_len=2),
    # absorbed chunked prefill over a cached prefix: 1024 new tokens per sequence over 4096
    # cached tokens, causal inside the chunk, paged cache (every new token a query sequence)
    "v3_chunk_b4_ctx4096_c1024": Workload("v3_chunk_b4_ctx4096_c1024", "decode_multi", B=4, H=128, d_model=0,
                                          d_c=512, d_hR=64, qk_nope=128, v_head=128, dtype="bf16",
                                          seed=_seed(7), ctx=4096, q_len=1024),
}

# the order the workloads are listed in (smallest first)
ORDER = ["tiny_fp32_layer", "v3_decode_b32_ctx4096", "v3_decode_fp8_b32_ctx4096", "v3_mtp_b32_ctx4096_q2",
         "v3_ragged_b64", "v3_chunk_b4_ctx4096_c1024",
         "v3_layer_b128_ctx8192", "v3_layer_folded_b128_ctx8192", "v2_prefill_b4_s4096"]


def shrink(w: Workload, **over) -> Workload:
    """A copy of `w` with some fields replaced (used for reduced-size parity cases)."""
    d = dict(w.__dict__)
    d.update(over)
    return Workload(**d)


def _tensor(w: Workload, name: str, shape, std: float) -> torch.Tensor:
    n = int(np.prod(shape))
    store = "bf16" if w.dtype == "bf16" else "f32"
    a = rng.normal(w.seed, TENSOR_IDS[name], n, std, store=store)
    t = torch.from_numpy(a.reshape(shape))
    return t.view(torch.bfloat16) if store == "bf16" else t


def lengths(w: Workload) -> np.ndarray:
    """Cached tokens per sequence before the decode step (int64 [B])."""
    if w.ctx_range is not None:
        return rng.randint(w.seed, TENSOR_IDS["lengths"], w.B, w.ctx_range[0], w.ctx_range[1])
    return np.full(w.B, w.ctx, dtype=np.int64)


def make_weights(w: Workload) -> Dict[str, torch.Tensor]:
    """Weights ~ N(0, 1/fan_in) in the storage type.

    Layouts (out x in, as a linear layer stores them):
      W_DKV [d_c, d_model], W_KR [d_hR, d_model], W_Q [H*(qk_nope+d_hR), d_model] head-major with
      the qk_nope rows of a head before its d_hR rows, W_UK [H, qk_nope, d_c],
      W_UV [H, v_head, d_c], W_O [d_model, H*v_head].
    """
    out = {
        "W_UK": _tensor(w, "W_UK", (w.H, w.qk_nope, w.d_c), 1.0 / math.sqrt(w.d_c)),
        "W_UV": _tensor(w, "W_UV", (w.H, w.v_head, w.d_c), 1.0 / math.sqrt(w.d_c)),
    }
    if w.kind in ("decode_layer", "prefill"):
        s = 1.0 / math.sqrt(w.d_model)
        out["W_DKV"] = _tensor(w, "W_DKV", (w.d_c, w.d_model), s)
        out["W_KR"] = _tensor(w, "W_KR", (w.d_hR, w.d_model), s)
        out["W_Q"] = _tensor(w, "W_Q", (w.H * (w.qk_nope + w.d_hR), w.d_model), s)
    if w.kind == "decode_layer":
        out["W_O"] = _tensor(w, "W_O", (w.d_model, w.H * w.v_head), 1.0 / math.sqrt(w.H * w.v_head))
    return out


def make_inputs(w: Workload) -> Dict[str, torch.Tensor]:
    """All inputs of one step of `w` as CPU tensors.

    decode_attn : cache [sum L, row], offsets int32 [B+1], q_nope [B,H,qk_nope],
                  q_rope [B,H,d_hR] (already rotated), W_UK, W_UV.
    decode_fp8  : as decode_attn (the bf16 rows are quantised to FP8 rows before the step).
    decode_multi: cache [sum (L + q_len), row] (the new tokens' rows last in each sequence),
                  offsets int32 [B+1], q_nope [B,q_len,H,qk_nope], q_rope [B,q_len,H,d_hR],
                  W_UK, W_UV.
    decode_layer: weights, h_new [B, d_model] (the token being decoded, at position L),
                  offsets int32 [B+1] over a cache of capacity L+1 per sequence, and either
                  h_hist [B, L, d_model] (cache built by appending at positions 0..L-1) or
                  cache [B*(L+1), row] with synthetic history rows.
    prefill     : weights, h [B, S, d_model].
    """
    d = make_weights(w)
    L = lengths(w)
    if w.kind in ("decode_attn", "decode_fp8"):
        offs = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
        d["offsets"] = torch.from_numpy(offs)
        d["cache"] = _tensor(w, "cache", (int(offs[-1]), w.row), w.cache_std)
        d["q_nope"] = _tensor(w, "q_nope", (w.B, w.H, w.qk_nope), 1.0)
        d["q_rope"] = _tensor(w, "q_rope", (w.B, w.H, w.d_hR), 1.0)
    elif w.kind == "decode_multi":
        offs = np.concatenate([[0], np.cumsum(L + w.q_len)]).astype(np.int32)
        d["offsets"] = torch.from_numpy(offs)
        d["cache"] = _tensor(w, "cache", (int(offs[-1]), w.row), w.cache_std)
        d["q_nope"] = _tensor(w, "q_nope", (w.B, w.q_len, w.H, w.qk_nope), 1.0)
        d["q_rope"] = _tensor(w, "q_rope", (w.B, w.q_len, w.H, w.d_hR), 1.0)
    elif w.kind == "decode_layer":
        cap = L + 1
        offs = np.concatenate([[0], np.cumsum(cap)]).astype(np.int32)
        d["offsets"] = torch.from_numpy(offs)
        d["h_new"] = _tensor(w, "h_new", (w.B, w.d_model), 1.0)
        if w.history == "hidden":
            d["h_hist"] = _tensor(w, "h_hist", (w.B, w.ctx, w.d_model), 1.0)
        else:
            d["cache"] = _tensor(w, "cache", (int(offs[-1]), w.row), w.cache_std)
    elif w.kind == "prefill":
        d["h"] = _tensor(w, "h", (w.B, w.ctx, w.d_model), 1.0)
    else:
        raise ValueError(w.kind)
    return d
