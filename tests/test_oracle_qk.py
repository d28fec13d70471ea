"""Pins of the oracle's maps-from-Q,K statement (compression without a dense map: MapFlow page
"MapFlow开源:大模型换班,Prefill为何能快20%?", section "存不下、读得慢?三个工程优化手段",
subsection 1).  The map is the sender's causal attention distribution; it is checked against
torch's scaled_dot_product_attention (a library routine computing the same softmax), a
hand-worked example, and invariants that a dropped term, a transposed operand or a wrong head
grouping would break."""
import math

import numpy as np
import pytest
import torch

import oracle


def _sdpa_probs(Q, K, L, scale):
    """Attention probabilities from torch SDPA: attending over V = identity returns them."""
    h_s, h_kv = Q.shape[1], K.shape[1]
    q = Q[:L].double().permute(1, 0, 2)                                   # [h_s, L, d]
    k = K[:L].double().repeat_interleave(h_s // h_kv, dim=1).permute(1, 0, 2)
    v = torch.eye(L, dtype=torch.float64).expand(h_s, L, L)
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale).numpy()


@pytest.mark.parametrize("L,h_s,h_kv,d,B", [(37, 4, 2, 16, 16), (70, 3, 1, 8, 32), (64, 2, 2, 32, 64)])
def test_qk_maps_match_sdpa(L, h_s, h_kv, d, B):
    g = torch.Generator().manual_seed(L * 7 + h_s)
    Q = torch.randn(L, h_s, d, generator=g).to(torch.bfloat16)
    K = torch.randn(L, h_kv, d, generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    A = oracle.qk_maps(Q, K, L, B, scale)
    Lp = -(-L // B) * B
    assert A.shape == (h_s, Lp, Lp)
    np.testing.assert_allclose(A[:, :L, :L], _sdpa_probs(Q, K, L, scale), rtol=1e-12, atol=1e-14)
    assert not A[:, L:, :].any() and not A[:, :, L:].any()          # padding
    assert not np.triu(A[:, :L, :L], 1).any()                         # causal


def test_qk_maps_hand_worked():
    """L = 3, one head, d = 1: q = (1, 2, 0.5), k = (1, -1, 2), scale 1.
    Row 1 weighs exp(2) against exp(-2); row 2 softmaxes (0.5, -0.5, 1)."""
    Q = torch.tensor([1.0, 2.0, 0.5]).reshape(3, 1, 1)
    K = torch.tensor([1.0, -1.0, 2.0]).reshape(3, 1, 1)
    A = oracle.qk_maps(Q, K, 3, 4, 1.0)[0]
    e = math.exp
    want = np.array([[1.0, 0, 0, 0],
                     [e(2) / (e(2) + e(-2)), e(-2) / (e(2) + e(-2)), 0, 0],
                     [e(0.5) / (e(0.5) + e(-0.5) + e(1)), e(-0.5) / (e(0.5) + e(-0.5) + e(1)),
                      e(1) / (e(0.5) + e(-0.5) + e(1)), 0],
                     [0, 0, 0, 0]])
    np.testing.assert_allclose(A, want, rtol=1e-14, atol=0)


def test_qk_maps_invariants():
    g = torch.Generator().manual_seed(3)
    L, h_s, h_kv, d = 50, 4, 2, 8
    Q = torch.randn(L, h_s, d, generator=g, dtype=torch.float64)
    K = torch.randn(L, h_kv, d, generator=g, dtype=torch.float64)
    A = oracle.qk_maps(Q, K, L, 16, 0.3)
    np.testing.assert_allclose(A[:, :L, :L].sum(axis=2), 1.0, rtol=1e-13)
    # a key shift c adds <q_i, c> to every score of row i: the distribution is unchanged
    c = torch.randn(1, h_kv, d, generator=g, dtype=torch.float64)
    A2 = oracle.qk_maps(Q, K + c, L, 16, 0.3)
    np.testing.assert_allclose(A2, A, rtol=1e-9, atol=1e-13)
    # query heads 0, 1 read key head 0 only: changing key head 1 leaves them alone
    K3 = K.clone()
    K3[:, 1] = torch.randn(L, d, generator=g, dtype=torch.float64) * 5
    A3 = oracle.qk_maps(Q, K3, L, 16, 0.3)
    np.testing.assert_array_equal(A3[:2], A[:2])
    assert np.abs(A3[2:] - A[2:]).max() > 1e-3
    # scale 0: uniform over the causal prefix
    A0 = oracle.qk_maps(Q, K, L, 16, 0.0)
    i = np.arange(L)
    np.testing.assert_allclose(A0[0, i, 0], 1.0 / (i + 1), rtol=1e-14)


def test_compress_qk_identity_map_is_attention():
    """tau = 1 keeps every causal block; with W = I the retrieval over the compressed maps is
    the sender's own causal attention output softmax(q k^T) V (torch SDPA with GQA)."""
    g = torch.Generator().manual_seed(11)
    L, h_s, h_kv, d, B = 45, 4, 2, 16, 16
    Q = torch.randn(L, h_s, d, generator=g).to(torch.bfloat16)
    K = torch.randn(L, h_kv, d, generator=g).to(torch.bfloat16)
    V = torch.randn(L, h_kv, 8, generator=g).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    r = oracle.compress_qk_seq(Q, K, L, B, 1.0, scale)
    W = np.eye(h_s, dtype=np.float32)
    outs = []
    for qb in range(-(-L // B)):
        kept = r["kept"][qb]
        assert kept.tolist() == list(range(qb + 1))
        hi = min(L, (qb + 1) * B) - qb * B
        outs.append(oracle.retrieve_block(r["values"][qb], kept, qb, B, W, V, h_kv, (0, hi)))
    O = np.concatenate(outs)
    q = Q.double().permute(1, 0, 2)
    k = K.double().repeat_interleave(2, dim=1).permute(1, 0, 2)
    v = V.double().repeat_interleave(2, dim=1).permute(1, 0, 2)
    want = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
    np.testing.assert_allclose(O, want.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)


def test_compress_qk_selection_follows_masses():
    """Masses of the float64 maps sum to the number of valid rows of the block row (each row of
    the map sums to 1), and selection walks them like any other map."""
    g = torch.Generator().manual_seed(5)
    L, h_s, h_kv, d, B = 100, 2, 1, 16, 16
    Q = (torch.randn(L, h_s, d, generator=g) * 2).to(torch.bfloat16)
    K = (torch.randn(L, h_kv, d, generator=g) * 2).to(torch.bfloat16)
    r = oracle.compress_qk_seq(Q, K, L, B, 0.8, 0.25)
    for qb, m in r["masses"].items():
        rows = min(L, (qb + 1) * B) - qb * B
        assert abs(m.sum() - h_s * rows) < 1e-9
        kept, _ = oracle.select(m, qb, 0.8)
        assert r["kept"][qb].tolist() == kept.tolist()
        assert m[kept].sum() >= 0.8 * m.sum() - 1e-12


def test_qk_slab_is_rows_of_the_maps():
    g = torch.Generator().manual_seed(9)
    L, B = 90, 32
    Q = torch.randn(L, 4, 16, generator=g).to(torch.bfloat16)
    K = torch.randn(L, 1, 16, generator=g).to(torch.bfloat16)
    A = oracle.qk_maps(Q, K, L, B, 0.25)
    for qb in range(3):
        np.testing.assert_array_equal(oracle.qk_slab(Q, K, L, B, qb, 0.25),
                                      A[:, qb * B:(qb + 1) * B, :(qb + 1) * B])
        m, kept, info, vals = oracle.compress_qk_row(Q, K, L, B, qb, 0.9, 0.25)
        r = oracle.compress_qk_seq(Q, K, L, B, 0.9, 0.25, rows=[qb])
        assert kept.tolist() == r["kept"][qb].tolist()
        np.testing.assert_array_equal(vals, r["values"][qb])
