"""The seeded input generator: determinism, shapes, storage rounding and planted structure."""
import numpy as np
import torch

from gen import WORKLOADS, cu_seqlens_of, dequantised, generate


def small(**kw):
    return WORKLOADS["llama8b_bf16_n8192"].with_(seqlens=(300, 0, 129), hq=4, hkv=2, **kw)


def test_deterministic_and_thread_independent():
    w = small()
    a = generate(w, workers=0)
    b = generate(w, workers=4)
    for key in ("q", "k", "v"):
        assert torch.equal(a[key].view(torch.int16), b[key].view(torch.int16))
    c = generate(w.with_(seed=1))
    assert not torch.equal(a["q"].view(torch.int16), c["q"].view(torch.int16))


def test_shapes_and_cu_seqlens():
    w = small()
    d = generate(w)
    assert d["q"].shape == (429, 4, 128) and d["k"].shape == (429, 2, 128)
    assert d["q"].dtype == torch.bfloat16
    assert list(d["cu_seqlens"]) == [0, 300, 300, 429]
    assert list(cu_seqlens_of([5, 7])) == [0, 5, 12]


def test_bf16_is_round_to_nearest_even_of_fp32():
    w = small()
    f = generate(w.with_(dtype="f32"))
    b = generate(w)
    assert torch.equal(f["q"].to(torch.bfloat16).view(torch.int16), b["q"].view(torch.int16))


def test_e4m3_per_head_absmax_maps_to_448():
    w = small(dtype="e4m3")
    f = generate(w.with_(dtype="f32"))
    e = generate(w)
    for name in ("q", "k", "v"):
        x, s = e[name], e[name[0] + "_scale"]
        amax = f[name].abs().amax(dim=(0, 2))
        assert torch.allclose(s, amax / 448.0)
        assert torch.allclose(x.to(torch.float32).abs().amax(dim=(0, 2)), torch.full_like(s, 448.0))
        deq = dequantised(x, s)
        rel = np.abs(deq - f[name].double().numpy()).max() / amax.max().item()
        assert rel < 2 ** -4


def test_sink_tokens_carry_the_sink_direction():
    # K tokens 0..3 of every sequence get +3u: their norm stands out from the noise (|k| ~ 1)
    w = small(dtype="f32")
    d = generate(w)
    k = d["k"]
    for a in (0, 300):
        head = k[a:a + 4].norm(dim=-1)
        rest = k[a + 4:a + 64].norm(dim=-1)
        assert head.min() > 2.0 and rest.median() < 2.0
