"""The on-disk format ("量化推理：INT8/INT4 ..." page: name.bin, name.scale, name.f32 and
manifest.json). The page checks that the persisted payload and scales decode to the
weights it evaluated; these tests check the same, plus the exact bytes of every file."""
import json
import os

import numpy as np
import pytest
import torch

import oracle


@pytest.fixture(scope="module")
def st():
    import int4_quantized_b200 as q4
    from int4_quantized_b200 import store

    q4.lib()
    return store


def packed(w, bits, group):
    p, s, status = oracle.pack(w, bits, group)
    assert status == oracle.OK
    return p, s


def test_round_trip_and_bytes(st, tmp_path):
    rng = np.random.default_rng(0)
    W1 = rng.normal(0, 0.05, (64, 32)).astype(np.float32)   # the page's W1 is [2D, H]
    W2 = rng.normal(0, 0.05, (32, 48)).astype(np.float32)
    E = rng.normal(0, 1, (10, 16)).astype(np.float32)
    q = {}
    for name, w, bits, g in (("W1", W1, 8, 32), ("W2", W2, 4, W2.size)):
        p, s = packed(w, bits, g)
        q[name] = st.QTensor(torch.from_numpy(p), torch.from_numpy(s), bits, g, w.shape)
    st.save(str(tmp_path), q, {"E": torch.from_numpy(E)})
    assert sorted(os.listdir(tmp_path)) == ["E.f32", "W1.bin", "W1.scale", "W2.bin", "W2.scale", "manifest.json"]
    # the files hold exactly what the page's code writes
    assert (tmp_path / "W1.bin").read_bytes() == q["W1"].payload.numpy().tobytes()
    assert (tmp_path / "W2.scale").read_bytes() == q["W2"].scales.numpy().astype("<f4").tobytes()
    assert (tmp_path / "E.f32").read_bytes() == E.astype("<f4").tobytes()
    man = (tmp_path / "manifest.json").read_text()
    assert man == json.dumps({"W1": {"bits": 8, "group": 32, "shape": [64, 32]},
                              "W2": {"bits": 4, "group": W2.size, "shape": [32, 48]}}, indent=2)
    lq, lp = st.load(str(tmp_path), shapes={"E": E.shape})
    for name in q:
        assert torch.equal(lq[name].payload, q[name].payload)
        assert torch.equal(lq[name].scales.view(torch.int32), q[name].scales.view(torch.int32))
        assert (lq[name].bits, lq[name].group, lq[name].shape) == (q[name].bits, q[name].group, q[name].shape)
    assert torch.equal(lp["E"], torch.from_numpy(E))


def test_folder_written_in_the_pages_format_decodes_to_the_same_weights(st, tmp_path):
    # written with plain NumPy file writes, as the page's loop does
    rng = np.random.default_rng(1)
    ws = {"a": (rng.normal(0, 0.1, (16, 64)).astype(np.float32), 4, 32),
          "b": (rng.normal(0, 0.1, (8, 24)).astype(np.float32), 8, 8),
          "c": (rng.normal(0, 0.1, (6, 10)).astype(np.float32), 4, 60)}
    manifest = {}
    for k, (w, bits, g) in ws.items():
        p, s = packed(w, bits, g)
        (tmp_path / f"{k}.bin").write_bytes(p.tobytes())
        (tmp_path / f"{k}.scale").write_bytes(s.astype("<f4").tobytes())
        manifest[k] = {"bits": bits, "group": g, "shape": list(w.shape)}
    (tmp_path / "manifest.json").write_text(json.dumps(manifest, indent=2))
    lq, lp = st.load(str(tmp_path))
    assert lp == {}
    for k, (w, bits, g) in ws.items():
        p, s = packed(w, bits, g)
        got = oracle.dequant(lq[k].payload.numpy(), lq[k].scales.numpy(), w.size, bits, g)
        want = oracle.dequant(p, s, w.size, bits, g)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32))


def test_mismatched_files_are_rejected(st, tmp_path):
    w = np.ones((4, 8), np.float32)
    p, s = packed(w, 4, 8)
    st.save(str(tmp_path), {"w": st.QTensor(torch.from_numpy(p), torch.from_numpy(s), 4, 8, (4, 8))})
    (tmp_path / "w.scale").write_bytes(s.astype("<f4").tobytes()[:-4])
    with pytest.raises(ValueError):
        st.load(str(tmp_path))
    with pytest.raises(ValueError):
        st.save(str(tmp_path), {"w": st.QTensor(torch.from_numpy(p), torch.from_numpy(s), 4, 16, (4, 8))})


@pytest.mark.gpu
def test_quantize_and_save_then_run_from_disk(st, tmp_path):
    import int4_quantized_b200 as q4

    rng = np.random.default_rng(2)
    shapes = {"q": (256, 512), "down": (512, 256), "norm": (512,)}
    host = {k: rng.normal(0, 0.02, s).astype(np.float32) for k, s in shapes.items()}
    dev = {k: torch.from_numpy(v).cuda() for k, v in host.items()}
    st.quantize_and_save(str(tmp_path / "int4_tensor"), {"q": dev["q"], "down": dev["down"], "norm": dev["norm"]},
                         4, None, keep=["norm"])
    st.quantize_and_save(str(tmp_path / "int8_g32"), {"q": dev["q"]}, 8, 32)
    for sub, bits, g in (("int4_tensor", 4, None), ("int8_g32", 8, 32)):
        lq, lp = st.load(str(tmp_path / sub), device="cuda", shapes={"norm": (512,)})
        for k, qt in lq.items():
            gg = host[k].size if g is None else g
            p, s = packed(host[k], bits, gg)
            assert np.array_equal(qt.payload.cpu().numpy(), p)
            deq = q4.qdequant(qt.payload, qt.scales, qt.shape, qt.bits, qt.group)
            want = oracle.dequant(p, s, host[k].size, bits, gg).reshape(qt.shape)
            assert np.array_equal(deq.cpu().numpy().view(np.uint32), want.view(np.uint32))
            N, K = qt.shape
            x = rng.normal(0, 1, (3, K)).astype(np.float32)
            y = q4.qgemm(torch.from_numpy(x).cuda(), qt.payload, qt.scales, N, K, qt.bits, qt.group)
            yref, bound = oracle.qgemm(x, p, s, N, K, bits, gg)
            assert np.all(np.abs(y.cpu().numpy().astype(np.float64) - yref) <= 1e-5 * bound + 1e-6)
        if sub == "int4_tensor":
            assert torch.equal(lp["norm"].cpu(), torch.from_numpy(host["norm"]))
