"""Expert parallelism across GPUs, emulated on one GPU: G ranks' buffers in
this GPU's memory, the library's EP kernels moving rows between them through
the same pointer tables a real group uses -- fused (moe_dispatch_route,
moe_ep_plan, moe_ep_dispatch storing each quantized copy at its owner,
moe_ep_combine_add_rmsnorm reading the owners' outputs) and two-step
(moe_dispatch, moe_ep_push, moe_ep_pull, moe_combine_add_rmsnorm).

Across G GPUs every GPU is one source of its own tokens, so the group's rows
must be exactly the single-GPU dispatch of all G * bs tokens (ordered by
instance, source, token, k; aclnnMoeDistributeDispatchV2, 计算公式), with GPU
q's receive buffer holding the stretch its instances own.  The tests compare
every receive buffer, its scales and copy ids, the receive counts and
offsets, every rank's global row of each copy, and the combine+Add+RMSNorm
output (aclnnMoeDistributeCombineAddRmsNorm, 计算公式) with the oracle run on
all G * bs tokens on one device.  Identity mapping tables keep the replica
choice out of the comparison (a GPU's update_expert numbers its own tokens)."""
import numpy as np
import pytest
import torch

from combine_moe_update_b200 import inputs as gen
from oracle import oracle as orc

from gpu_harness import assert_close_bf16, dev, dev_bf16, host, poison_

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_moe_update_b200 import binding
    return binding


@pytest.fixture(scope="module")
def EP():
    from combine_moe_update_b200 import ep
    return ep


def _bytes(a, lo, hi):
    a = np.ascontiguousarray(a)
    return a.view(np.uint8).reshape(a.shape[0], -1)[lo:hi]


def _inputs(seed, G, bs, H, E, K, ws, smooth):
    rng = np.random.Generator(np.random.PCG64([81, seed]))
    T = G * bs
    return dict(
        x=gen.bf16_bits(rng.standard_normal((T, H), np.float32)),
        ids=gen.topk_uniform(rng, T, E, K),
        scales=gen.softmax_scales(rng, T, K),
        residual=gen.bf16_bits(rng.standard_normal((T, H), np.float32)),
        shared=gen.bf16_bits(rng.standard_normal((T, H), np.float32)),
        gamma=gen.bf16_bits(rng.uniform(0.5, 1.5, size=H).astype(np.float32)),
        expert_rows=gen.bf16_bits(rng.standard_normal((T * K, H), np.float32)),  # by global row
        smooth=rng.uniform(0.5, 2.0, size=(E, H)).astype(np.float32) if smooth else None,
        table=gen.identity_table(E, ws))


@pytest.mark.parametrize("G,bs,H,E,K,ws,mode,smooth", [
    (2, 64, 1024, 16, 4, 4, 0, False),
    (4, 48, 2048, 32, 6, 8, 2, True),
    (2, 40, 1040, 32, 8, 8, 3, False),    # ragged last tile
    (4, 32, 1024, 64, 8, 16, 4, False),   # mxfp8
    (8, 24, 7168, 256, 8, 32, 2, True),   # the decode row length, eight GPUs
    (2, 512, 1024, 16, 8, 2, 1, True),    # static per-instance scales, 4096 copies per GPU
    (2, 512, 2048, 64, 16, 8, 3, False),  # 8192 copies per GPU, per-tile int8
])
@pytest.mark.parametrize("fused", [True, False], ids=["fused", "two_step"])
def test_emulated_group_equals_one_gpu_dispatch(B, EP, G, bs, H, E, K, ws, mode, smooth, fused):
    _check_group(B, EP, G, bs, H, E, K, ws, mode, smooth, fused)


@pytest.mark.parametrize("G,bs,H,E,K,ws,mode,smooth", [
    (2, 256, 2048, 32, 8, 8, 2, True),   # smooth scales, two copy groups per token
    (2, 40, 1024, 16, 8, 4, 2, True),    # four copy groups per token
    (2, 64, 1024, 16, 6, 4, 0, False),   # one quantization per token
])
@pytest.mark.parametrize("fused", [True, False], ids=["fused", "two_step"])
def test_emulated_group_with_pruned_tokens(B, EP, G, bs, H, E, K, ws, mode, smooth, fused):
    """A pruning threshold above many tokens' largest routing weight: tokens
    with no sent copy (and copy groups with none) must still record their
    copies' global rows as -1, so the combine sums nothing for them."""
    _check_group(B, EP, G, bs, H, E, K, ws, mode, smooth, fused, prune=0.3, min_unsent_tokens=1)


def _check_group(B, EP, G, bs, H, E, K, ws, mode, smooth, fused, prune=0.0, min_unsent_tokens=0):
    inp = _inputs(G * 1000 + mode, G, bs, H, E, K, ws, smooth or mode == 1)
    grp = EP.EmulatedGroup(G, fused=fused, bs=bs, hidden=H, top_k=K, num_instances=E, ep_world_size=ws,
                           quant_mode=mode)
    for r in grp.ranks:
        for t in r.buffers() + [r.global_idx, r.recv_counts, r.recv_offsets]:
            if t is not None:
                poison_(t)
    sm = None if inp["smooth"] is None else dev(inp["smooth"])
    table = dev(inp["table"])
    sl = lambda a, g: np.ascontiguousarray(a[g * bs:(g + 1) * bs])
    grp.dispatch([dict(expert_ids=dev(sl(inp["ids"], g)), table=table, x=dev_bf16(sl(inp["x"], g)),
                       expert_scales=dev(sl(inp["scales"], g)), smooth=sm, prune_threshold=prune)
                  for g in range(G)])
    torch.cuda.synchronize()
    for r in grp.ranks:
        assert r.device_errors() == 0

    # the oracle: all G * bs tokens on one device
    bal, bm, _ = orc.update_expert(inp["ids"], inp["table"], ws, expert_scales=inp["scales"],
                                   prune_threshold=prune)
    od = orc.dispatch(inp["x"], bal, E, mode, mask=bm, smooth=inp["smooth"])
    assert ((od["expand_idx"] < 0).all(axis=1)).sum() >= min_unsent_tokens
    off, El = od["offsets"], E // G
    for q, r in enumerate(grp.ranks):
        b, e_ = int(off[q * El]), int(off[(q + 1) * El])
        np.testing.assert_array_equal(host(r.recv_counts), od["counts"][q * El:(q + 1) * El])
        np.testing.assert_array_equal(host(r.recv_offsets), off[q * El:(q + 1) * El + 1] - b)
        np.testing.assert_array_equal(_bytes(host(r.recv_x), 0, e_ - b), _bytes(od["expand_x"], b, e_))
        np.testing.assert_array_equal(host(r.recv_src)[:e_ - b], od["src_of_row"][b:e_])
        if od["dyn_scales"] is not None:
            np.testing.assert_array_equal(_bytes(host(r.recv_scales), 0, e_ - b), _bytes(od["dyn_scales"], b, e_))
        np.testing.assert_array_equal(host(r.global_idx), od["expand_idx"][q * bs:(q + 1) * bs])

    # the expert step: each GPU's output rows are the synthetic rows of its global rows
    for q, r in enumerate(grp.ranks):
        b, e_ = int(off[q * El]), int(off[(q + 1) * El])
        poison_(r.expert_out)
        r.expert_out[:e_ - b].copy_(dev_bf16(inp["expert_rows"][b:e_]))
    outs = grp.combine([dict(expert_scales=dev(sl(inp["scales"], g)), residual=dev_bf16(sl(inp["residual"], g)),
                             gamma=dev_bf16(inp["gamma"]), norm_eps=1e-6, shared_x=dev_bf16(sl(inp["shared"], g)))
                        for g in range(G)])
    torch.cuda.synchronize()
    oc = orc.combine_add_rmsnorm(inp["expert_rows"], od["expand_idx"], inp["scales"], inp["residual"],
                                 inp["gamma"], 1e-6, shared_x=inp["shared"])
    for g, (r, o) in enumerate(zip(grp.ranks, outs)):
        assert r.device_errors() == 0
        assert_close_bf16(host(o["y"]), oc["y_f64"][g * bs:(g + 1) * bs], what=f"y of GPU {g}")


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "two_step"])
def test_receive_buffer_too_small_is_flagged(B, EP, fused):
    G, bs, H, E, K, ws = 2, 64, 1024, 16, 4, 4
    inp = _inputs(7, G, bs, H, E, K, ws, False)
    grp = EP.EmulatedGroup(G, fused=fused, bs=bs, hidden=H, top_k=K, num_instances=E, ep_world_size=ws,
                           quant_mode=0, recv_rows=16)
    for r in grp.ranks:
        poison_(r.recv_x)
    sl = lambda a, g: np.ascontiguousarray(a[g * bs:(g + 1) * bs])
    grp.dispatch([dict(expert_ids=dev(sl(inp["ids"], g)), table=dev(inp["table"]), x=dev_bf16(sl(inp["x"], g)))
                  for g in range(G)])
    torch.cuda.synchronize()
    bal, bm, _ = orc.update_expert(inp["ids"], inp["table"], ws)
    od = orc.dispatch(inp["x"], bal, E, 0, mask=bm)
    for q, r in enumerate(grp.ranks):
        assert r.device_errors() & B.DEV_CAPACITY
        b = int(od["offsets"][q * (E // G)])
        # the rows that fit are right; nothing past the buffer was written (it has 16 rows)
        np.testing.assert_array_equal(_bytes(host(r.recv_x), 0, 16), _bytes(od["expand_x"], b, b + 16))


def test_ep_combine_flags_a_row_outside_the_group(B, EP):
    """A global row past the group's last row is reported (MOE_DEV_BAD_ID)
    and that copy is dropped from the sum, as a pruned copy."""
    G, bs, H, E, K, ws = 2, 32, 1024, 16, 4, 4
    inp = _inputs(11, G, bs, H, E, K, ws, False)
    grp = EP.EmulatedGroup(G, bs=bs, hidden=H, top_k=K, num_instances=E, ep_world_size=ws, quant_mode=0)
    sl = lambda a, g: np.ascontiguousarray(a[g * bs:(g + 1) * bs])
    grp.dispatch([dict(expert_ids=dev(sl(inp["ids"], g)), table=dev(inp["table"]), x=dev_bf16(sl(inp["x"], g)))
                  for g in range(G)])
    bal, bm, _ = orc.update_expert(inp["ids"], inp["table"], ws)
    od = orc.dispatch(inp["x"], bal, E, 0, mask=bm)
    total = int(od["offsets"][-1])
    off, El = od["offsets"], E // G
    for q, r in enumerate(grp.ranks):
        b, e_ = int(off[q * El]), int(off[(q + 1) * El])
        r.expert_out[:e_ - b].copy_(dev_bf16(inp["expert_rows"][b:e_]))
    idx = od["expand_idx"].copy()
    grp.ranks[0].global_idx[0, 0] = total  # one past the group's rows
    idx[0, 0] = -1
    outs = grp.combine([dict(expert_scales=dev(sl(inp["scales"], g)), residual=dev_bf16(sl(inp["residual"], g)),
                             gamma=dev_bf16(inp["gamma"]), norm_eps=1e-6) for g in range(G)])
    torch.cuda.synchronize()
    assert grp.ranks[0].device_errors() & B.DEV_BAD_ID
    assert grp.ranks[1].device_errors() == 0
    oc = orc.combine_add_rmsnorm(inp["expert_rows"], idx, inp["scales"], inp["residual"], inp["gamma"], 1e-6)
    for g, o in enumerate(outs):
        assert_close_bf16(host(o["y"]), oc["y_f64"][g * bs:(g + 1) * bs], what=f"y of GPU {g}")


def test_ep_dispatch_refuses_parameters_that_disagree(B, EP):
    """moe_ep_dispatch checks the dispatch parameters against the EP ones."""
    G, bs, H, E, K, ws = 2, 16, 1024, 16, 4, 4
    grp = EP.EmulatedGroup(G, bs=bs, hidden=H, top_k=K, num_instances=E, ep_world_size=ws, quant_mode=0)
    r = grp.ranks[0]
    x = torch.zeros((bs, H), dtype=torch.bfloat16, device="cuda")
    bad = B.ep_params(bs, K, E, G, 0, H, 0, r.cap)  # mode 0 rows are 2H bytes
    with pytest.raises(B.MoeError):
        B.ep_dispatch(bad, x, r.bal, ws, 0, r.route_out, grp.tables.recv_x, None, None, r.global_idx, r.ep_ws)
    bad = B.ep_params(bs, K, E, G, 0, 2 * H, 4, r.cap)  # mode 0 sends no scales
    with pytest.raises(B.MoeError):
        B.ep_dispatch(bad, x, r.bal, ws, 0, r.route_out, grp.tables.recv_x, grp.tables.recv_x, None,
                      r.global_idx, r.ep_ws)


def test_process_group_ep_one_rank(B, EP):
    """ProcessGroupEP on a one-GPU NCCL group (the counts gathered by
    all_gather_into_tensor, the barriers as all-reduces, fused dispatch and
    combine through the group's pointer tables) equals the oracle."""
    import datetime
    import socket
    import torch.distributed as dist
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    bs, H, E, K, ws = 96, 2048, 32, 6, 8
    inp = _inputs(5, 1, bs, H, E, K, ws, True)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        grp = EP.ProcessGroupEP(bs=bs, hidden=H, top_k=K, num_instances=E, ep_world_size=ws, quant_mode=2)
        r = grp.r
        grp.dispatch(expert_ids=dev(inp["ids"]), table=dev(inp["table"]), x=dev_bf16(inp["x"]),
                     expert_scales=dev(inp["scales"]), smooth=dev(inp["smooth"]))
        bal, bm, _ = orc.update_expert(inp["ids"], inp["table"], ws, expert_scales=inp["scales"])
        od = orc.dispatch(inp["x"], bal, E, 2, mask=bm, smooth=inp["smooth"])
        n = int(od["offsets"][-1])
        torch.cuda.synchronize()
        assert r.received() == n
        np.testing.assert_array_equal(_bytes(host(r.recv_x), 0, n), _bytes(od["expand_x"], 0, n))
        np.testing.assert_array_equal(_bytes(host(r.recv_scales), 0, n), _bytes(od["dyn_scales"], 0, n))
        np.testing.assert_array_equal(host(r.global_idx), od["expand_idx"])
        r.expert_out[:n].copy_(dev_bf16(inp["expert_rows"][:n]))
        out = grp.combine(expert_scales=dev(inp["scales"]), residual=dev_bf16(inp["residual"]),
                          gamma=dev_bf16(inp["gamma"]), norm_eps=1e-6, shared_x=dev_bf16(inp["shared"]))
        torch.cuda.synchronize()
        assert r.device_errors() == 0
        oc = orc.combine_add_rmsnorm(inp["expert_rows"], od["expand_idx"], inp["scales"], inp["residual"],
                                     inp["gamma"], 1e-6, shared_x=inp["shared"])
        assert_close_bf16(host(out["y"]), oc["y_f64"], what="y")
        grp.close()
    finally:
        dist.destroy_process_group()
