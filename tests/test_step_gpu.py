"""Graph-captured decode steps (sparse_long_context_ffd_b200.step): the replayed
graph must reproduce the eager fused steps bit for bit, and the stand-in
attention layer must match a plain PyTorch layer in dense mode."""
import numpy as np
import pytest
import torch

import ffd_workloads as fw
from gpu_util import to_dev_bf16
from sparse_long_context_ffd_b200 import ffd
from sparse_long_context_ffd_b200.step import DecodeStep, StandInAttentionLayer

pytestmark = pytest.mark.gpu


def _setup(seed, T=64, B=2, G=4, Hkv=2, cap=2048, S=4):
    w = fw.random_small_workload(seed, B, G, Hkv, cap, T, S, 2.0, cap // 2, cap - 8, needles=1)
    inp = fw.make_inputs(w)
    shape = ffd.make_shape(w.batch, w.num_q_heads, w.num_kv_heads, w.capacity, T, S)
    return w, inp, shape


@pytest.mark.parametrize("fmt", ["int4", "tr"])
def test_graph_step_equals_eager_fused_steps(fmt):
    w, inp, shape = _setup(90)
    start = (inp["lengths"] - 6).astype(np.int32)
    k_g, v_g = to_dev_bf16(inp["k"]), to_dev_bf16(inp["v"])
    k_e, v_e = k_g.clone(), v_g.clone()
    len_g = torch.from_numpy(start.copy()).cuda()
    len_e = torch.from_numpy(start.copy()).cuda()
    step = DecodeStep(shape, k_g, v_g, len_g, 2.0, fmt=fmt, advance=True)
    eager = ffd.ThumbResidBuffers(shape) if fmt == "tr" else ffd.DecodeBuffers(shape)
    if fmt == "tr":
        ffd.quantize_keys_tr(shape, k_e, len_e, 0, eager.k_thumb, eager.k_resid, eager.k_scales)
    else:
        ffd.quantize_keys(shape, k_e, len_e, 0, eager.k_packed, eager.k_scales)
    rng = np.random.default_rng(7)
    for i in range(6):
        q = fw.f32_to_bf16_bits(rng.standard_normal((w.batch, w.num_q_heads, 128)).astype(np.float32))
        pos = start + i  # the new token's position (length after the step - 1)
        kn = np.stack([inp["k"][b, :, pos[b]] for b in range(w.batch)])
        vn = np.stack([inp["v"][b, :, pos[b]] for b in range(w.batch)])
        step.host_q.copy_(torch.from_numpy(q.view(np.int16)).view(torch.bfloat16))
        step.host_k_new.copy_(torch.from_numpy(kn.view(np.int16)).view(torch.bfloat16))
        step.host_v_new.copy_(torch.from_numpy(vn.view(np.int16)).view(torch.bfloat16))
        step.step()
        len_e.add_(1)
        qd, knd, vnd = to_dev_bf16(q), to_dev_bf16(kn), to_dev_bf16(vn)
        if fmt == "tr":
            ffd.decode_append_tr(shape, qd, knd, vnd, k_e, v_e, eager.k_thumb, eager.k_resid,
                                 eager.k_scales, len_e, 2.0, eager.out, eager.mask, eager.workspace)
        else:
            ffd.decode_append(shape, qd, knd, vnd, k_e, v_e, eager.k_packed, eager.k_scales, len_e,
                              2.0, eager.out, eager.mask, eager.workspace)
        torch.cuda.synchronize()
        assert torch.equal(step.host_out.view(torch.int16), eager.out.cpu().view(torch.int16)), i
        assert torch.equal(step.host_mask, eager.mask.cpu()), i
    assert torch.equal(len_g, len_e)
    assert torch.equal(k_g.view(torch.int16), k_e.view(torch.int16))
    assert torch.equal(v_g.view(torch.int16), v_e.view(torch.int16))
    assert step.check() == 0


def test_stand_in_layer_matches_torch_layer_in_dense_mode():
    w, inp, shape = _setup(91, B=2, G=4, Hkv=2, cap=1024)
    hidden = 512
    start = (inp["lengths"] - 3).astype(np.int32)
    k, v = to_dev_bf16(inp["k"]), to_dev_bf16(inp["v"])
    k_ref, v_ref = k.clone(), v.clone()
    lengths = torch.from_numpy(start.copy()).cuda()
    layer = StandInAttentionLayer(shape, hidden, k, v, lengths, float("inf"), seed=3)
    B, Hq, Hkv, G = w.batch, w.num_q_heads, w.num_kv_heads, w.group
    n = start.copy()
    rng = np.random.default_rng(11)
    for i in range(3):
        x = torch.from_numpy(rng.standard_normal((B, hidden)).astype(np.float32)).to(torch.bfloat16)
        layer.host_x.copy_(x)
        layer.step()
        # plain layer: the same bf16 projections, fp32 attention over the cache
        xd = x.cuda()
        q = torch.matmul(xd, layer.w_q).view(B, Hq, 128)
        kn = torch.matmul(xd, layer.w_k).view(B, Hkv, 128)
        vn = torch.matmul(xd, layer.w_v).view(B, Hkv, 128)
        for b in range(B):
            k_ref[b, :, n[b]] = kn[b]
            v_ref[b, :, n[b]] = vn[b]
        n += 1
        att = torch.zeros((B, Hq, 128), device="cuda")
        for b in range(B):
            kk = k_ref[b, :, :n[b]].float().repeat_interleave(G, 0)
            vv = v_ref[b, :, :n[b]].float().repeat_interleave(G, 0)
            att[b] = torch.nn.functional.scaled_dot_product_attention(
                q[b].float()[:, None], kk, vv)[:, 0]
        y_ref = torch.matmul(att.to(torch.bfloat16).view(B, -1), layer.w_o).float().cpu()
        err = (layer.host_y.float() - y_ref).abs().max().item()
        assert err <= 2e-2 * max(1.0, y_ref.abs().max().item()), (i, err)
    assert torch.equal(lengths.cpu(), torch.from_numpy(n))
    for b in range(B):  # the appended projections are in the cache
        diff = (k[b, :, :n[b]].float() - k_ref[b, :, :n[b]].float()).abs().max().item()
        assert diff <= 1e-2 * max(1.0, k_ref[b, :, :n[b]].float().abs().max().item())
    assert layer.core.check() == 0
