"""Checkpoint / resume: a handle exported mid-stream and imported into a fresh
handle continues bit for bit like the original (outputs of every later chunk,
across a RoPE refresh and with the re-pinned sink, and the final cache), for
the bf16 and the e4m3 cache; malformed or foreign checkpoints are refused and
leave the target unchanged."""
import numpy as np
import pytest
import torch

from gpu_harness import Runner
from inputgen.workloads import Workload
from rolling_kv_cache_sa_b200._lib import SA_ERR_INVALID_ARG, SA_SINK_REPIN, SAError

pytestmark = pytest.mark.gpu

CK = Workload("ckpt_bf16_8x16", B=2, H=4, D=128, fh=8, fw=16, C=2, S=1, W=4, n_chunks=10,
              dtype="bf16", refresh_period=4, starts=(0, 3))


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")


@pytest.mark.parametrize("w", [CK, CK.with_(name="ckpt_e4m3", cache="e4m3",
                                            fp8_scales=((1.5, 2.0, 0.5, 4.0),
                                                        (2.0, 1.0, 3.0, 0.25),
                                                        (1.0, 8.0, 0.5, 2.0)))],
                         ids=lambda w: w.name)
def test_export_import_continues_bit_for_bit(w):
    a = Runner(w)
    a.cache.set_sink_mode(SA_SINK_REPIN)
    b = None
    try:
        cut = 5
        for g in range(cut):
            a.step(g)
        torch.cuda.synchronize()
        blob = a.cache.export()
        b = Runner(w.with_(fp8_scales=()))  # the scales come with the checkpoint
        b.cache.import_(blob)
        for s in range(w.B):
            assert b.cache.state(s) == a.cache.state(s)
        for g in range(cut, w.n_steps):
            chunks, active = a.step(g)
            b.step(g)
            torch.cuda.synchronize()
            for s, c in enumerate(chunks):
                if c >= 0:
                    assert torch.equal(a.out[s], b.out[s]), (g, s)
        for s in range(w.B):
            ka, va = a.cache.copy_out(s)
            kb, vb = b.cache.copy_out(s)
            np.testing.assert_array_equal(ka, kb)
            np.testing.assert_array_equal(va, vb)
        assert a.device_status() == 0 and b.device_status() == 0
    finally:
        a.close()
        if b is not None:
            b.close()


def test_foreign_or_damaged_checkpoints_are_refused():
    a = Runner(CK)
    other = Runner(CK.with_(name="ckpt_other", H=2))
    try:
        for g in range(3):
            a.step(g)
        torch.cuda.synchronize()
        blob = a.cache.export()
        before = [other.cache.state(s) for s in range(CK.B)]
        # another configuration (H = 2), and a truncated copy
        for bad in (blob, blob[:-1]):
            with pytest.raises(SAError) as e:
                other.cache.import_(bad)
            assert e.value.status == SA_ERR_INVALID_ARG
        assert [other.cache.state(s) for s in range(CK.B)] == before
        same = Runner(CK.with_(name="ckpt_same"))
        try:
            damaged = blob.copy()
            damaged[:8] = np.frombuffer(b"NOTACKPT", np.uint8)
            with pytest.raises(SAError):
                same.cache.import_(damaged)
            assert [same.cache.state(s) for s in range(CK.B)] == [(0, 0)] * CK.B
        finally:
            same.close()
    finally:
        a.close()
        other.close()
