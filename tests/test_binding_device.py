"""The binding runs every library call with the device of the problem's
tensors current (the C library launches on the current device and would
otherwise address another GPU's memory), and takes the default stream of
that device.  Host-only: the library and ``torch.cuda.device`` are replaced
by recording fakes, and the tensors live on the ``meta`` device, so no GPU
is needed to see which device each call runs under."""
import contextlib
import ctypes

import pytest
import torch

from block_sparse_attention_psa_b200 import psa

B, H, N, d = 1, 2, 256, 64
M = N // 64
META = torch.device("meta")


class _RecordingLib:
    """Stands in for the loaded library: every entry point records the device
    that was current when it was called and returns PSA_OK."""

    def __init__(self, log, current):
        self._log, self._current = log, current

    def psa_workspace_size(self, *args):
        return 1 << 16

    def psa_route_capacity(self, B, H, M, causal):
        return B * H * M * M

    def __getattr__(self, name):
        def entry(*args):
            self._log.append((name, self._current[-1] if self._current else None))
            return psa.PSA_OK
        return entry


@pytest.fixture
def recorded(monkeypatch):
    log, current = [], []

    @contextlib.contextmanager
    def fake_device(dev):
        current.append(torch.device(dev))
        try:
            yield
        finally:
            current.pop()

    streams = []

    def fake_stream(stream, like):
        streams.append(like.device)
        return ctypes.c_void_p(0)

    monkeypatch.setattr(torch.cuda, "device", fake_device)
    monkeypatch.setattr(psa, "lib", lambda: _RecordingLib(log, current))
    monkeypatch.setattr(psa, "_ptr", lambda t: None if t is None else ctypes.c_void_p(1 << 20))
    monkeypatch.setattr(psa, "_stream", fake_stream)
    return log, streams


def _meta(*shape, dtype=torch.float32):
    return torch.empty(*shape, dtype=dtype, device=META)


def test_every_entry_point_runs_with_the_tensors_device_current(recorded):
    log, streams = recorded
    q, k, v = (_meta(B, H, N, d, dtype=torch.bfloat16) for _ in range(3))
    qbar, kbar, vsum = psa.psa_pool(q, k, v)
    for route in (psa.psa_route_topk, psa.psa_route_thresh, psa.psa_route_thresh_prob):
        route(qbar, kbar, 0.5)
    rp = _meta(B * H * M + 1, dtype=torch.int32)
    ci = _meta(B * H * M * M, dtype=torch.int32)
    ws = psa.workspace(B, H, N, d, META)
    psa.psa_attn(q, k, v, kbar, vsum, rp, ci, ws=ws, want_lse=True)
    psa.psa_dense(q, k, v, ws=ws)
    psa.psa_attn_noalloc(q, k, v, kbar, vsum, rp, ci)
    psa.psa_read_status(ws)
    psa.psa_read_fixup_count(ws)
    called = [name for name, _ in log]
    assert called == ["psa_pool", "psa_route_topk", "psa_route_thresh", "psa_route_thresh_prob", "psa_attn",
                      "psa_dense", "psa_attn_noalloc", "psa_read_status", "psa_read_fixup_count"]
    for name, dev in log:
        assert dev == META, f"{name} ran with {dev} current, the tensors live on {META}"
    assert streams and all(s == META for s in streams)
