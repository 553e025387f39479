"""moe_dispatch_noalloc: dispatch for callers that cannot allocate device memory.

Some callers only get to hand the library the tensors it reads and writes --
a runtime with a fixed memory plan, or a host framework that gives a custom
op no workspace -- so they cannot provide moe_dispatch's workspace.
moe_dispatch_noalloc keeps that workspace in a static array inside the
library instead.  These tests call it through the C ABI twice in a row and
require exactly the bytes moe_dispatch produces for the same inputs (dispatch
outputs are compared bit for bit everywhere in this suite), plus its error
word, which must start from zero on every call.

This file is collected last on purpose, and passes both on its own in a fresh
process and after the other tests.
"""
import numpy as np
import pytest
import torch

from combine_moe_update_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_moe_update_b200 import binding
    return binding


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def dev_bf16(bits):
    return dev(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16)


def as_bytes(t, rows):
    return t.view(torch.uint8).reshape(t.shape[0], -1)[:rows].cpu().numpy()


@pytest.mark.parametrize("name", ["deepseek_decode_bs512", "skewed_eplb", "max_shape", "tiny"])
def test_noalloc_matches_dispatch_twice(B, name):
    w = gen.make(name)
    ws = B.new_workspace()
    bal, bm = B.update_expert(dev(w.expert_ids), dev(w.table), w.ep_world_size,
                              expert_scales=dev(w.expert_scales), prune_threshold=w.prune_threshold,
                              workspace=ws)
    x = dev_bf16(w.x)
    sm = None if w.smooth is None else dev(w.smooth)
    ref = B.dispatch(x, bal, w.num_instances, w.ep_world_size, w.quant_mode, mask=bm, smooth=sm, workspace=ws)
    torch.cuda.synchronize()
    n = int(ref["offsets"][-1].item())
    for call in range(2):
        out = B.alloc_dispatch_outputs(w.bs, w.hidden, w.top_k, w.num_instances, w.quant_mode)
        for v in out.values():
            if v is not None:
                v.view(torch.uint8).fill_(0xA5)
        err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        B.dispatch_noalloc(x, bal, w.num_instances, w.ep_world_size, w.quant_mode, mask=bm, smooth=sm,
                           out=out, device_error=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"call {call}: device error {int(err.item())}"
        assert torch.equal(out["expand_idx"], ref["expand_idx"])
        assert torch.equal(out["counts"], ref["counts"])
        assert torch.equal(out["offsets"], ref["offsets"])
        assert torch.equal(out["src_of_row"][:n], ref["src_of_row"][:n])
        np.testing.assert_array_equal(as_bytes(out["expand_x"], n), as_bytes(ref["expand_x"], n))
        if w.quant_mode != 0:
            np.testing.assert_array_equal(as_bytes(out["dyn_scales"], n), as_bytes(ref["dyn_scales"], n))


def test_noalloc_error_word_starts_from_zero_each_call(B):
    w = gen.make("tiny")
    ids = w.expert_ids.copy()
    ids[1, 0] = w.num_instances + 5  # out of range: dropped and reported
    x = dev_bf16(w.x)
    err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    B.dispatch_noalloc(x, dev(ids), w.num_instances, w.ep_world_size, 0, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == B.DEV_BAD_ID
    B.dispatch_noalloc(x, dev(w.expert_ids), w.num_instances, w.ep_world_size, 0, device_error=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_noalloc_rejects_bad_sizes_before_launch(B):
    x = torch.zeros((513, 1024), dtype=torch.bfloat16, device="cuda")  # Bs beyond 512
    ids = torch.zeros((513, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.dispatch_noalloc(x, ids, 8, 4, 0)
    assert e.value.status == B.MOE_ERR_INVALID_ARG


def test_noalloc_refuses_calls_that_need_a_route_table(B):
    """Several source ranks past 8192 copies need a workspace larger than the
    static array (the route's slice table): the call is refused with
    MOE_ERR_WORKSPACE and nothing is enqueued, so the outputs keep their
    poison."""
    S, bs, H, K, E, ws = 2, 512, 1024, 16, 64, 8
    rng = np.random.Generator(np.random.PCG64(90))
    x = dev_bf16(gen.bf16_bits(rng.standard_normal((S * bs, H), np.float32)))
    ids = dev(gen.topk_uniform(rng, S * bs, E, K))
    assert B.dispatch_workspace_bytes(bs, H, K, ws, E, 0, 0, S) > 256
    out = B.alloc_dispatch_outputs(S * bs, H, K, E, 0)
    for v in out.values():
        if v is not None:
            v.view(torch.uint8).fill_(0xA5)
    torch.cuda.synchronize()
    with pytest.raises(B.MoeError) as e:
        B.dispatch_noalloc(x, ids, E, ws, 0, out=out, sources=S)
    assert e.value.status == B.MOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    for k, v in out.items():
        if v is not None:
            assert bool((v.view(torch.uint8) == 0xA5).all()), k
