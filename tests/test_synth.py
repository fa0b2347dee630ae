"""The seeded cache generator: determinism, layout and the concentrated-centre structure."""
import numpy as np
import torch

import synth
from synth.gen import layer_heads


def _derotate(K, pos, theta=1e6, d=128):
    F = d // 2
    w = np.power(theta, -2.0 * np.arange(F) / d)
    a = pos[:, None].astype(np.float64) * w[None, :]
    kr, ki = K[:, :F].astype(np.float64), K[:, F:].astype(np.float64)
    return kr * np.cos(a) + ki * np.sin(a), ki * np.cos(a) - kr * np.sin(a)


def test_contig_is_seeded_and_concentrated():
    wl = synth.WORKLOADS["single_layer_4k"]
    a = synth.make_contig(wl, "cpu")
    b = synth.make_contig(wl, "cpu")
    assert torch.equal(a.K.view(torch.int16), b.K.view(torch.int16))
    assert torch.equal(a.V.view(torch.int16), b.V.view(torch.int16))
    assert a.n_rows == 8 and a.total == 8 * 4096
    np.testing.assert_array_equal(a.row_off_np, np.arange(9) * 4096)
    heads = layer_heads(wl, 0, "cpu")
    for r in (0, 5):
        lo, hi = a.row_off_np[r], a.row_off_np[r + 1]
        K = a.K[lo:hi].float().numpy()
        pr, pi = _derotate(K, a.pos[lo:hi].numpy())
        _, _, h = a.row_lhs(r)
        mu_r, mu_i = heads.key_re[h].numpy(), heads.key_im[h].numpy()
        sc = heads.key_scale[h].numpy()
        # sample mean within a few standard errors of the centre, spread ~ r|mu|
        assert np.all(np.abs(pr.mean(0) - mu_r) < 6 * sc / np.sqrt(4096) + 0.02 * np.abs(mu_r) + 1e-2)
        ratio = np.sqrt(((pi - mu_i) ** 2).mean(0)) / sc
        assert 0.9 < ratio.mean() < 1.1
    assert a.qcal.shape == (1, 32, 1024, 128)


def test_zero_centre_heads_are_pure_noise():
    wl = synth.WORKLOADS["sweep_b64_adversarial"]
    z = wl.zero_centre_pairs()
    assert z.sum() == round(0.05 * z.size)
    layer = int(np.nonzero(z.any(axis=1))[0][0])
    heads = layer_heads(wl, layer, "cpu")
    h = int(np.nonzero(z[layer])[0][0])
    assert float(heads.key_re[h].abs().max()) == 0.0 and float(heads.key_scale[h].min()) > 0
    G = wl.group
    assert float(heads.q_re[h * G:(h + 1) * G].abs().max()) == 0.0


def test_paged_layout_matches_contig_rows():
    wl = synth.WORKLOADS["paged_16seq"].with_(batch=3, seq_len=(40, 70))
    p = synth.make_paged(wl, "cpu")
    lens = p.lens
    bs = wl.block_size
    used = set()
    for s, n in enumerate(lens):
        nb = (int(n) + bs - 1) // bs
        blocks = p.block_table_np[s, :nb]
        assert np.all(blocks >= 0)
        used.update(blocks.tolist())
        for h in range(wl.n_kv_heads):
            j = np.arange(n)
            pos = p.pos[torch.as_tensor(blocks[j // bs]), torch.as_tensor(j % bs), h].numpy()
            np.testing.assert_array_equal(pos, j)
    assert len(used) == sum((int(n) + bs - 1) // bs for n in lens)


def test_seq_lengths_in_range():
    wl = synth.WORKLOADS["sweep_b64"]
    L = wl.seq_lengths()
    assert L.shape == (64,) and L.min() >= 4096 and L.max() <= 65536
    np.testing.assert_array_equal(L, wl.seq_lengths())


def test_fp8_conversion_is_nearest_e4m3_of_the_clamped_value():
    """to_fp8: every value becomes the e4m3 code nearest to it after clamping to
    +-448, a tie between two representable values going to the code with the even
    mantissa - checked by exhaustive search over the finite codes, decoded with the
    oracle's definition of the format."""
    import numpy as np
    import torch

    import oracle
    import synth

    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_bits_to_f64(codes)
    finite = ~np.isnan(vals)
    cv, cc = vals[finite], codes[finite]
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(4000) * np.exp(rng.uniform(-12, 7, 4000)),
                        [0.0, 448.0, -448.0, 1000.0, -1e9, 2.0 ** -10, 2.0 ** -9 * 1.5, 1.0625, 3.0 * 2.0 ** -9]])
    x = x.astype(np.float32).astype(np.float64)  # the generator converts from fp32
    got = synth.to_fp8(torch.tensor(x, dtype=torch.float32)).view(torch.uint8).numpy()
    got_v = oracle.e4m3_bits_to_f64(got)
    xc = np.clip(x, -448.0, 448.0)
    for xi, gi, gv in zip(xc, got, got_v):
        d = np.abs(cv - xi)
        near = np.unique(cv[d == d.min()])
        assert gv in near, (xi, gi, near)
        if len(near) == 2:  # an exact tie between two values: the even mantissa wins
            assert gi & 1 == 0, (xi, gi, near)


def test_fp8_conversion_in_chunks_is_the_one_shot_conversion():
    """The chunked conversion (bounded temporary memory for caches near the device's
    size) gives the same bytes as converting the whole tensor at once, including
    values beyond the e4m3 range (clamped to +-448) and a ragged last chunk."""
    import torch
    g = torch.Generator().manual_seed(7)
    t = (torch.randn(1001, 37, generator=g) * 200).to(torch.bfloat16)
    t[0, :4] = torch.tensor([1e4, -1e4, 448.0, -0.0], dtype=torch.bfloat16)
    whole = t.float().clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    got = synth.to_fp8(t, chunk=1000)
    assert got.shape == t.shape and got.dtype == torch.float8_e4m3fn
    assert torch.equal(got.view(torch.uint8), whole.view(torch.uint8))
