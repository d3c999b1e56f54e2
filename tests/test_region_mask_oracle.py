"""Pins of the oracle's optional shifted-window region mask.

The mask is the usual one of shifted-window attention: on the map rolled by
-s, rows fall into three bands (before the last window, the last window's
part before the wrap-around, the wrapped-around part) and columns alike; a
query attends only to keys of its own (row band, column band) region.  The
pins tie `region_labels` to a label image built by slicing the rolled map,
and masked attention to plain attention over each region's tokens alone.
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import rib_oracle as R

rng = np.random.default_rng(4321)


def rnd(*shape, std=1.0):
    return rng.standard_normal(shape) * std


def sliced_label_image(H, W, M, s):
    """Label image of the rolled map: consecutive integers over the 3 x 3
    grid of (row slice, column slice), row slices outermost."""
    img = np.zeros((H, W), dtype=np.int64)
    if s == 0:
        return img
    cnt = 0
    for hs in (slice(0, H - M), slice(H - M, H - s), slice(H - s, H)):
        for ws in (slice(0, W - M), slice(W - M, W - s), slice(W - s, W)):
            img[hs, ws] = cnt
            cnt += 1
    return img


@pytest.mark.parametrize("H,W,M,s", [(32, 32, 16, 8), (48, 32, 16, 8), (64, 48, 16, 4),
                                     (192, 192, 96, 48), (32, 32, 16, 0)])
def test_region_labels_match_sliced_label_image(H, W, M, s):
    img = sliced_label_image(H, W, M, s)
    for wy in range(H // M):
        for wx in range(W // M):
            want = img[wy * M:(wy + 1) * M, wx * M:(wx + 1) * M].reshape(-1)
            np.testing.assert_array_equal(O.region_labels(H, W, M, s, wy, wx), want)


def test_region_labels_counts_in_the_corner_window():
    # the last window of a map shifted by half a window holds four regions of
    # (M/2)^2 tokens each; every other window holds one region
    H = W = 64
    M, s = 16, 8
    lab = O.region_labels(H, W, M, s, H // M - 1, W // M - 1)
    assert sorted(np.bincount(lab)[np.bincount(lab) > 0].tolist()) == [64, 64, 64, 64]
    assert len(set(O.region_labels(H, W, M, s, 0, 0).tolist())) == 1
    assert len(set(O.region_labels(H, W, M, s, H // M - 1, 0).tolist())) == 2


def _unit(N, d=8, r=4):
    return rnd(N, d), rnd(N, d), rnd(N, d), rnd(N, r), rnd(N, r)


def test_masked_forward_equals_attention_within_each_region():
    H = W = 32
    M, s = 16, 8
    N = M * M
    qc, kc, v, qp, kp = _unit(N)
    scale = 0.3
    lab = O.region_labels(H, W, M, s, 1, 1)
    out, lse = O.attention_unit(qc, kc, v, qp, kp, scale, labels=lab)
    for g in np.unique(lab):
        idx = np.nonzero(lab == g)[0]
        # plain attention over the region's tokens only, through torch SDPA
        q = torch.tensor(np.concatenate([qc[idx], qp[idx]], 1))[None, None]
        k = torch.tensor(np.concatenate([kc[idx], kp[idx]], 1))[None, None]
        vv = torch.tensor(v[idx])[None, None]
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, vv, scale=scale)[0, 0]
        np.testing.assert_allclose(out[idx], ref.numpy(), rtol=1e-12, atol=1e-12)
        sc = scale * (np.concatenate([qc[idx], qp[idx]], 1) @ np.concatenate([kc[idx], kp[idx]], 1).T)
        m = sc.max(1)
        np.testing.assert_allclose(lse[idx], m + np.log(np.exp(sc - m[:, None]).sum(1)),
                                   rtol=1e-12, atol=1e-12)


def test_masked_backward_equals_backward_within_each_region():
    H = W = 32
    M, s = 16, 8
    N = M * M
    qc, kc, v, qp, kp = _unit(N)
    dout = rnd(N, 8)
    scale = 0.3
    lab = O.region_labels(H, W, M, s, 1, 1)
    g = O.attention_unit_backward(qc, kc, v, qp, kp, scale, dout, labels=lab)
    for reg in np.unique(lab):
        idx = np.nonzero(lab == reg)[0]
        # torch autograd on the region's tokens alone
        t = [torch.tensor(a[idx], requires_grad=True) for a in (qc, kc, v, qp, kp)]
        q = torch.cat([t[0], t[3]], 1)
        k = torch.cat([t[1], t[4]], 1)
        p = torch.softmax(scale * q @ k.T, dim=1)
        (p @ t[2] * torch.tensor(dout[idx])).sum().backward()
        for got, ref in zip((g[0], g[1], g[2], g[3], g[4]),
                            (t[0].grad, t[1].grad, t[2].grad, t[3].grad, t[4].grad)):
            np.testing.assert_allclose(got[idx], ref.numpy(), rtol=1e-10, atol=1e-12)


def test_map_level_mask_changes_only_border_windows():
    B, H, W, heads, d, r = 1, 32, 48, 1, 8, 4
    M, s = 16, 8
    qkv = rnd(B, H, W, 3, heads, d)
    qp, kp = rnd(heads, M, M, r), rnd(heads, M, M, r)
    o0, l0 = O.attn_fwd(qkv, M, s, qp, kp, scale=0.3)
    o1, l1 = O.attn_fwd(qkv, M, s, qp, kp, scale=0.3, region_mask=True)
    # pixels whose rolled position lies in an interior window keep their result
    rolled_y = (np.arange(H) - s) % H
    rolled_x = (np.arange(W) - s) % W
    interior = (rolled_y[:, None] < H - M) & (rolled_x[None, :] < W - M)
    np.testing.assert_array_equal(o0[0][interior], o1[0][interior])
    assert np.abs(o0[0][~interior] - o1[0][~interior]).max() > 1e-3
    # without a shift the mask is empty
    o2, _ = O.attn_fwd(qkv, M, 0, qp, kp, scale=0.3, region_mask=True)
    o3, _ = O.attn_fwd(qkv, M, 0, qp, kp, scale=0.3)
    np.testing.assert_array_equal(o2, o3)


# -------------------------------------------------- planted mistakes (on the CPU)

def _labels_off_by_one(H, W, M, s, wy, wx):
    def band(pos, size):
        if s == 0:
            return np.zeros_like(pos)
        return np.where(pos < size - M, 0, np.where(pos < size - s - 1, 1, 2))
    i, j = np.divmod(np.arange(M * M), M)
    return 3 * band(wy * M + i, H) + band(wx * M + j, W)


def _labels_rows_only(H, W, M, s, wy, wx):
    lab = _orig_labels(H, W, M, s, wy, wx)
    return lab // 3


def _allowed_ignores_mask(labels, r0, r1, rows=None):
    return None


_orig_labels = R.region_labels


@pytest.mark.parametrize("name,bad,pins", [
    ("region_labels", _labels_off_by_one, [test_region_labels_match_sliced_label_image]),
    ("region_labels", _labels_rows_only, [test_region_labels_match_sliced_label_image,
                                          test_region_labels_counts_in_the_corner_window]),
    ("_allowed", _allowed_ignores_mask, [test_masked_forward_equals_attention_within_each_region,
                                         test_masked_backward_equals_backward_within_each_region]),
])
def test_planted_mask_mistake_is_caught(monkeypatch, name, bad, pins):
    monkeypatch.setattr(R, name, bad)
    if name == "region_labels":
        monkeypatch.setattr(O, name, bad)
    caught = 0
    for pin in pins:
        try:
            if pin is test_region_labels_match_sliced_label_image:
                pin(32, 32, 16, 8)
            else:
                pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"{name}: planted mistake not caught"
