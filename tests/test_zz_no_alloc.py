"""mla_decode_absorbed_noalloc: the decode entry point for callers that cannot allocate
device memory (engines that own all GPU memory through their own pool, code where
allocation is forbidden).  Its scratch is a fixed array inside the library, so it takes no
workspace.  It must give the same results as mla_decode_absorbed with a caller workspace,
also on a second call that finds the previous call's data left in the shared scratch.

This file is collected last on purpose: it runs after every other test, and must also
pass alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from helpers import assert_close
from test_gpu_parity import dims_of, reduced_attn_inputs

pytestmark = pytest.mark.gpu

mla = pytest.importorskip("compressed_kv_cache_absorbed_b200")


@pytest.mark.parametrize("lengths", [[300, 1, 77, 513, 0, 64], [4096, 4096, 129, 2]])
def test_noalloc_matches_the_workspace_entry_point(lengths):
    w, inp = reduced_attn_inputs(lengths, seed=23)
    g = {k: v.cuda() for k, v in inp.items()}
    dims = dims_of(w)
    B = w.B
    assert mla.mla_decode_workspace_size(dims, B) <= (64 << 20)
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
    ref = torch.empty(B, w.H, w.v_head, dtype=torch.bfloat16, device="cuda")
    ws = mla.workspace(mla.mla_decode_workspace_size(dims, B))
    mla.mla_decode_absorbed(dims, weights, g["cache"], g["offsets"], ref, ws, q_nope=g["q_nope"],
                            q_rope=g["q_rope"])
    # a larger, different batch first, so that its data is what the checked calls find left
    # in the shared scratch
    wb, ib = reduced_attn_inputs([2000] * 24, seed=29)
    gb = {k: v.cuda() for k, v in ib.items()}
    ob = torch.empty(wb.B, wb.H, wb.v_head, dtype=torch.bfloat16, device="cuda")
    mla.mla_decode_absorbed_noalloc(dims, weights, gb["cache"], gb["offsets"], ob, q_nope=gb["q_nope"],
                                    q_rope=gb["q_rope"])
    outs = []
    for _ in range(2):   # the second call finds the first call's data in the scratch
        o = torch.full((B, w.H, w.v_head), float("nan"), dtype=torch.bfloat16, device="cuda")
        mla.mla_decode_absorbed_noalloc(dims, weights, g["cache"], g["offsets"], o, q_nope=g["q_nope"],
                                        q_rope=g["q_rope"])
        outs.append(o)
    assert mla.mla_get_device_error() == (0, 0)
    r = ref.cpu()
    for o in outs:
        assert_close(o.cpu(), r.double(), "bf16", "no-alloc vs workspace entry point")
    weights.close()


def test_noalloc_rejects_batches_beyond_its_scratch():
    w, inp = reduced_attn_inputs([1], seed=5)
    dims = dims_of(w)
    big = 4096
    assert mla.mla_decode_workspace_size(dims, big) > (64 << 20)
    g = {k: v.cuda() for k, v in inp.items()}
    weights = mla.mla_absorb_weights(dims, g["W_UK"], g["W_UV"])
    offs = torch.zeros(big + 1, dtype=torch.int32, device="cuda")
    q = torch.zeros(big, w.H, w.qk_nope, dtype=torch.bfloat16, device="cuda")
    qr = torch.zeros(big, w.H, w.d_hR, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(big, w.H, w.v_head, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mla.MLAError) as e:
        mla.mla_decode_absorbed_noalloc(dims, weights, g["cache"], offs, out, q_nope=q, q_rope=qr)
    assert e.value.status == mla.MLA_ERR_WORKSPACE
    assert torch.all(out == 0)
    weights.close()
