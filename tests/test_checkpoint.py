"""Checkpoint and resume (CPU): the training state round-trips bit for bit,
and damaged files are refused."""
import os

import numpy as np
import pytest

from spatiotemporal_neural_field_b200 import checkpoint as ck
from spatiotemporal_neural_field_b200 import synthetic as S

torch = pytest.importorskip("torch")


def _state():
    grid, mlp = S.GRID_SPORTS, S.MLP_SPORTS
    t16 = S.hash_tables(grid, scale=1.0)
    rng = np.random.default_rng(1)
    return {
        "tables_f16": torch.from_numpy(t16),
        "tables_f32": torch.from_numpy(t16.astype(np.float32)),
        "weights_f32": torch.from_numpy(S.mlp_weights(mlp).astype(np.float32)),
        "adam_m": torch.from_numpy(rng.standard_normal(1000).astype(np.float32)),
        "adam_v": rng.random(1000).astype(np.float32),
        "empty": np.zeros((0, 3), np.float32),
    }


def test_round_trip(tmp_path):
    state = _state()
    meta = {"grid": {"L": 16, "F": 2, "log2_T": 19}, "note": "sports frame"}
    p = str(tmp_path / "ck.bin")
    ck.save(p, state, step=42, meta=meta)
    assert not os.path.exists(p + ".tmp")
    got, step, m = ck.load(p)
    assert step == 42 and m == meta
    assert list(got) == list(state)
    for k, v in state.items():
        want = v.numpy() if hasattr(v, "numpy") else v
        assert got[k].dtype == want.dtype and got[k].shape == want.shape, k
        assert np.array_equal(got[k].view(np.uint8), want.view(np.uint8)), k
    # every blob starts on a 64-byte boundary
    import json
    import struct
    with open(p, "rb") as f:
        f.read(8)
        (hlen,) = struct.unpack("<Q", f.read(8))
        hdr = json.loads(f.read(hlen))
    assert all(e["offset"] % 64 == 0 for e in hdr["tensors"])
    # to a device given as torch tensors (CPU here)
    got_t, _, _ = ck.load(p, device="cpu")
    assert torch.equal(got_t["tables_f16"], state["tables_f16"])


def test_damaged_files_are_refused(tmp_path):
    state = _state()
    p = str(tmp_path / "ck.bin")
    ck.save(p, state, step=1)
    raw = bytearray(open(p, "rb").read())
    # a flipped byte inside the first tensor fails its CRC
    import json
    import struct
    (hlen,) = struct.unpack("<Q", raw[8:16])
    first = json.loads(bytes(raw[16:16 + hlen]))["tensors"][0]
    bad = bytearray(raw)
    bad[first["offset"] + 5] ^= 0x40
    q = str(tmp_path / "bad.bin")
    open(q, "wb").write(bad)
    with pytest.raises(ck.CheckpointError, match="CRC"):
        ck.load(q)
    # a truncated file
    open(q, "wb").write(raw[:len(raw) // 2])
    with pytest.raises(ck.CheckpointError):
        ck.load(q)
    # not a checkpoint
    open(q, "wb").write(b"NOTSPIN4" + raw[8:])
    with pytest.raises(ck.CheckpointError, match="not a spin4d"):
        ck.load(q)
    # another format version
    hdr = json.loads(bytes(raw[16:16 + hlen]))
    hdr["version"] = 9
    h2 = json.dumps(hdr, sort_keys=True).encode()
    assert len(h2) == hlen
    open(q, "wb").write(raw[:16] + h2 + raw[16 + hlen:])
    with pytest.raises(ck.CheckpointError, match="version"):
        ck.load(q)


def test_resume_continues_adam_exactly(tmp_path):
    """Three oracle Adam steps straight through equal two steps, a save and
    load of (params, m, v, step), then the third: the state carries everything."""
    from oracle import decoder as dec
    rng = np.random.default_rng(3)
    p0 = rng.standard_normal(500)
    grads = [rng.standard_normal(500) for _ in range(3)]
    p, m, v = p0, np.zeros(500), np.zeros(500)
    for i, g in enumerate(grads):
        p, m, v = dec.adam_step(p, g, m, v, i + 1, 1e-3, 0.9, 0.99, 1e-15)
    q, mq, vq = p0, np.zeros(500), np.zeros(500)
    for i, g in enumerate(grads[:2]):
        q, mq, vq = dec.adam_step(q, g, mq, vq, i + 1, 1e-3, 0.9, 0.99, 1e-15)
    path = str(tmp_path / "adam.bin")
    ck.save(path, {"params": q, "m": mq, "v": vq}, step=2)
    st, step, _ = ck.load(path)
    q, _, _ = dec.adam_step(st["params"], grads[2], st["m"], st["v"], step + 1, 1e-3, 0.9, 0.99, 1e-15)
    assert np.array_equal(q, p)
