"""One sender serving several receivers (the one-sender, several-receivers workflow of the MapFlow
page "MapFlow开源:大模型换班,Prefill为何能快20%?", section "它能做什么:三种典型工作流").

mf_map_retrieve_multi must give, bit for bit, what mf_map_retrieve gives receiver by receiver,
whether the receivers share launches or not; one receiver of each case is also checked against
the oracle within the bf16 tolerance (max-abs 2e-2, relative-L2 1e-2)."""
import dataclasses

import numpy as np
import pytest
import torch

import cross_model_attention_mf_b200 as mf
import synth
from synth import device as sdev
from tests.gpu_common import assert_O_close, check_rows, run_compress

pytestmark = pytest.mark.gpu


def _status_ok():
    rc, bits = mf.mf_get_status()
    assert rc == mf.MF_OK and bits == 0, (rc, bits)


def _sender(lens, n_layers=1, B=64, h_s=32):
    w = synth.Workload("multi", lens, B=B, h_s=h_s, h_r=32, h_kv=8, d=128, dtype="bf16",
                       tau=0.95, n_heavy=16, reading=3, n_sender_layers=n_layers,
                       n_receiver_layers=n_layers, page_size=16)
    bsrs, packs = [], []
    for l in range(n_layers):
        pack = sdev.fill_maps(sdev.alloc_maps(w), w, l)
        bsrs.append(run_compress(w, pack))
        packs.append(pack)
    _status_ok()
    return w, bsrs, packs


def _receiver(w, h_r, h_kv, seed, layer_map, paged=False):
    """A receiver with its own head map, V (seeded apart from the others) and layer map."""
    wr = dataclasses.replace(w, h_r=h_r, h_kv=h_kv, seed=seed, n_receiver_layers=len(layer_map))
    W = sdev.w_weights(wr)
    V = torch.stack([sdev.v_contiguous(wr, l) for l in range(len(layer_map))])
    r = mf.Receiver(list(layer_map), W, V, h_r, h_kv, v_layer_stride=V[0].numel())
    if paged:
        parts = [sdev.v_paged(wr, V[l]) for l in range(len(layer_map))]
        Vp = torch.stack([p[0] for p in parts])
        r = mf.Receiver(list(layer_map), W, Vp, h_r, h_kv, paged=(parts[0][1], w.page_size),
                        v_layer_stride=Vp[0].numel())
    return wr, r, V


def _one_by_one(w, bsrs, r):
    qbase = sdev.qblock_base(w)
    return mf.mf_map_retrieve(bsrs, r.layer_map, r.W, r.V, _cu(w), _cu(w), qbase, max(w.lens),
                              r.h_r, r.h_kv, total_q=w.tokens, paged=r.paged,
                              v_layer_stride=r.v_layer_stride)


def _cu(w):
    return torch.tensor(np.concatenate([[0], np.cumsum(w.lens)]), dtype=torch.int32, device="cuda")


def _multi(w, bsrs, rs):
    return mf.mf_map_retrieve_multi(bsrs, rs, _cu(w), _cu(w), sdev.qblock_base(w), max(w.lens),
                                    total_q=w.tokens)


def _fused(w, bsrs, rs):
    return mf.mf_retrieve_multi_fused(bsrs, rs, _cu(w), _cu(w), sdev.qblock_base(w), max(w.lens),
                                      total_q=w.tokens)


def _oracle_check(w, packs, bsrs, wr, r, V, layer):
    """Receiver r, receiver layer `layer`, against the oracle on every row."""
    from tests.test_gpu_parity import _all_rows, _oracle_O_all
    s_layer = r.layer_map[layer]
    orows, nb = check_rows(w, packs[s_layer], bsrs[s_layer], _all_rows(w))
    assert nb == 0
    want = _oracle_O_all(wr, orows, r.W[layer].cpu().numpy(), V[layer].cpu())
    return want


def test_three_receivers_share_launches():
    """Receivers with 32 / 8, 24 / 8 (GQA 3) and 8 / 2 heads, one of them on paged V."""
    w, bsrs, packs = _sender((300, 129, 64, 1))
    specs = [(32, 8, 11, False), (24, 8, 12, True), (8, 2, 13, False)]
    made = [_receiver(w, h_r, h_kv, seed, [0], paged) for h_r, h_kv, seed, paged in specs]
    rs = [m[1] for m in made]
    assert _fused(w, bsrs, rs) == 1
    outs = _multi(w, bsrs, rs)
    _status_ok()
    for r, O in zip(rs, outs):
        assert torch.equal(O, _one_by_one(w, bsrs, r))
    wr, r, V = made[1]
    want = _oracle_check(w, packs, bsrs, wr, r, V, 0)
    assert_O_close(outs[1][0].float().cpu().numpy(), want, "bf16", "receiver 1 (gq 3, paged)")
    _status_ok()


def test_six_receivers_two_layers():
    """Six receivers (two launches per layer step) over two sender layers mapped [1, 0]."""
    w, bsrs, packs = _sender((200, 77, 130), n_layers=2)
    made = [_receiver(w, 16, 4, 20 + k, [1, 0], paged=(k % 2 == 1)) for k in range(6)]
    rs = [m[1] for m in made]
    assert _fused(w, bsrs, rs) == 1
    outs = _multi(w, bsrs, rs)
    _status_ok()
    for r, O in zip(rs, outs):
        assert torch.equal(O, _one_by_one(w, bsrs, r))
    assert not torch.equal(outs[0], outs[2])  # receivers differ
    wr, r, V = made[4]
    want = _oracle_check(w, packs, bsrs, wr, r, V, 1)
    assert_O_close(outs[4][1].float().cpu().numpy(), want, "bf16", "receiver 4, layer 1")
    _status_ok()


def test_receivers_that_cannot_share_run_one_by_one():
    """A GQA-8 receiver takes the SIMT kernel: the receivers then run one after another."""
    w, bsrs, packs = _sender((190, 64))
    made = [_receiver(w, 32, 8, 31, [0]), _receiver(w, 32, 4, 32, [0])]
    rs = [m[1] for m in made]
    assert _fused(w, bsrs, rs) == 0
    outs = _multi(w, bsrs, rs)
    _status_ok()
    for r, O in zip(rs, outs):
        assert torch.equal(O, _one_by_one(w, bsrs, r))
    wr, r, V = made[1]
    want = _oracle_check(w, packs, bsrs, wr, r, V, 0)
    assert_O_close(outs[1][0].float().cpu().numpy(), want, "bf16", "gq 8 receiver")
    _status_ok()
