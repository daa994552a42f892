"""The Python binding's marshalling, on the CPU, against a stand-in library.

Every entry point of ``nonlinear_rnn_solve_newton_b200`` is called with
correctly shaped tensors: each must reach exactly its C function.  Wrongly
shaped outputs, status words and info structs must be refused before the call.
The stand-in library records calls and returns success, and the device
requirement of the argument checks is lifted for the test; dtype, shape and
contiguity are still checked.  The real library, its kernels and the
no-CPU-path guarantee are tested elsewhere (tests/test_abi.py, the GPU suites).
"""
import contextlib
from types import SimpleNamespace

import pytest
import torch

import nonlinear_rnn_solve_newton_b200 as pr


class _FakeLib:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append(name)
            return 4096 if name == "pararnn_workspace_size" else 0
        return fn


def _check_host(name, t, dtype, shape):
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


@pytest.fixture
def fake(monkeypatch):
    lib = _FakeLib()
    monkeypatch.setattr(pr, "load", lambda build_if_missing=True: lib)
    monkeypatch.setattr(pr, "_check_dev", _check_host)
    monkeypatch.setattr(pr, "_workspace",
                        lambda n, device, stream=None: torch.empty(n, dtype=torch.uint8))
    monkeypatch.setattr(pr, "_stream_handle", lambda s, dev=None: None)
    monkeypatch.setattr(pr, "_one_device", lambda **named: torch.device("cpu"))
    monkeypatch.setattr(pr, "_device_guard", lambda dev: contextlib.nullcontext())
    pr._ws_sizes.clear()
    yield lib
    pr._ws_sizes.clear()   # sizes from the stand-in must not outlive the test


B, L, D, K = 2, 5, 8, 16
f32 = torch.float32


def z(*shape, dtype=f32):
    return torch.zeros(shape, dtype=dtype)


def info_t():
    return z(pr.INFO_BYTES // 4, dtype=torch.int32)


def status_t():
    return z(1, dtype=torch.int32)


def test_every_entry_point_reaches_its_c_function(fake):
    cases = [
        ("pararnn_scan_diag", lambda: pr.scan_diag(z(B, L, D), z(B, L, D), z(B, D),
                                                   status=status_t())),
        ("pararnn_scan_block2", lambda: pr.scan_block2(z(B, L, D, 2, 2), z(B, L, D, 2),
                                                       z(B, D, 2), status=status_t())),
        ("pararnn_solve_gru", lambda: pr.solve_gru(z(B, L, 3, D), z(3, D), z(B, D),
                                                   info=info_t())),
        ("pararnn_solve_gru", lambda: pr.solve_gru(z(B, L, 3, D, dtype=torch.bfloat16),
                                                   z(3, D))),
        ("pararnn_solve_lstm", lambda: pr.solve_lstm(z(B, L, 4, D), z(4, D), z(B, D), z(B, D))),
        ("pararnn_solve_gru_noalloc", lambda: pr.solve_gru_noalloc(z(B, L, 3, D), z(3, D))),
        ("pararnn_solve_mhgru", lambda: pr.solve_mhgru(z(B, L, 3, D), z(3, D // 8, 8, 8))),
        ("pararnn_solve_mhgru_strided",
         lambda: pr.solve_mhgru_strided(z(B, L, 3, D), z(3, D // 8, 8, 8),
                                        z(D // 8, dtype=torch.int32))),
        ("pararnn_solve_gru_backward",
         lambda: pr.solve_gru_backward(z(B, L, 3, D), z(3, D), z(B, L, D), z(B, L, D), z(B, D),
                                       status=status_t())),
        ("pararnn_solve_lstm_backward",
         lambda: pr.solve_lstm_backward(z(B, L, 4, D), z(4, D), z(B, L, D), z(B, L, D),
                                        z(B, L, D), None,
                                        out=(z(B, L, 4, D), z(4, D), z(B, D), z(B, D)))),
        ("pararnn_step_gru", lambda: pr.step_gru(z(B, 3, D), z(3, D), z(B, D))),
        ("pararnn_step_lstm", lambda: pr.step_lstm(z(B, 4, D), z(4, D), z(B, D), z(B, D))),
        ("pararnn_rollout_gru", lambda: pr.rollout_gru(z(B, L, 3, D), z(3, D), z(B, D))),
        ("pararnn_rollout_lstm", lambda: pr.rollout_lstm(z(B, L, 4, D), z(4, D))),
        ("pararnn_rollout_mhgru", lambda: pr.rollout_mhgru(z(B, L, 3, D), z(3, D // 8, 8, 8))),
        ("pararnn_step_mhgru", lambda: pr.step_mhgru(z(B, 3, D), z(3, D // 8, 8, 8), z(B, D))),
        ("pararnn_solve_gru_projected",
         lambda: pr.solve_gru_projected(z(B, L, K, dtype=torch.bfloat16),
                                        z(3 * D, K, dtype=torch.bfloat16), z(3 * D), z(3, D),
                                        z(B, D), info=info_t())),
        ("pararnn_input_projection",
         lambda: pr.input_projection(z(B, L, K, dtype=torch.bfloat16),
                                     z(3 * D, K, dtype=torch.bfloat16), z(3 * D),
                                     status=status_t())),
    ]
    for name, call in cases:
        fake.calls.clear()
        call()
        assert [c for c in fake.calls if c != "pararnn_workspace_size"] == [name], name


def test_outputs_status_and_info_are_checked_before_the_call(fake):
    bad = [
        # LSTM backward outputs of the wrong shape
        lambda: pr.solve_lstm_backward(z(B, L, 4, D), z(4, D), z(B, L, D), z(B, L, D),
                                       z(B, L, D), None,
                                       out=(z(B, L, 3, D), z(4, D), z(B, D), z(B, D))),
        lambda: pr.solve_lstm_backward(z(B, L, 4, D), z(4, D), z(B, L, D), z(B, L, D),
                                       z(B, L, D), None,
                                       out=(z(B, L, 4, D), z(4, D), z(B, D), z(B, D + 1))),
        # GRU backward output of the wrong shape
        lambda: pr.solve_gru_backward(z(B, L, 3, D), z(3, D), z(B, L, D), z(B, L, D),
                                      out=(z(B, L, 3, D), z(3, D), z(B + 1, D))),
        # status words: wrong dtype or size
        lambda: pr.scan_diag(z(B, L, D), z(B, L, D), status=z(1)),
        lambda: pr.scan_block2(z(B, L, D, 2, 2), z(B, L, D, 2), status=z(2, dtype=torch.int32)),
        lambda: pr.solve_gru_backward(z(B, L, 3, D), z(3, D), z(B, L, D), z(B, L, D),
                                      status=z(1, dtype=torch.int64)),
        lambda: pr.input_projection(z(B, K, dtype=torch.bfloat16),
                                    z(3 * D, K, dtype=torch.bfloat16), status=z(1)),
        # info structs: too small or the wrong dtype
        lambda: pr.solve_gru(z(B, L, 3, D), z(3, D), info=z(4, dtype=torch.int32)),
        lambda: pr.solve_lstm(z(B, L, 4, D), z(4, D), info=z(pr.INFO_BYTES // 4)),
        lambda: pr.solve_mhgru(z(B, L, 3, D), z(3, D // 8, 8, 8),
                               info=z(pr.INFO_BYTES, dtype=torch.uint8)),
        lambda: pr.solve_gru_noalloc(z(B, L, 3, D), z(3, D), info=z(1, dtype=torch.int32)),
        # solve outputs
        lambda: pr.solve_gru(z(B, L, 3, D), z(3, D), out=z(B, L + 1, D)),
        lambda: pr.solve_lstm(z(B, L, 4, D), z(4, D), out=(z(B, L, D), z(B, L, D, dtype=torch.float64))),
    ]
    for i, call in enumerate(bad):
        fake.calls.clear()
        with pytest.raises((ValueError, TypeError)):
            call()
        assert [c for c in fake.calls if c != "pararnn_workspace_size"] == [], i


def _on(dev):
    """A stand-in for a CUDA tensor on `dev` (only what the device check reads)."""
    return SimpleNamespace(is_cuda=dev is not None,
                           device=torch.device("cuda", dev) if dev is not None else
                           torch.device("cpu"))


def test_one_device_accepts_one_device_and_skips_absent_arguments():
    assert pr._one_device(P=_on(1), a=_on(1), h0=None, out=_on(1)) == torch.device("cuda", 1)


def test_one_device_refuses_mixed_devices():
    # the C library launches on the current device: a tensor on another GPU
    # would be read through peer memory or fault, so the binding refuses it
    with pytest.raises(ValueError, match="one device"):
        pr._one_device(P=_on(1), a=_on(0))
    with pytest.raises(ValueError, match="one device"):
        pr._one_device(P=_on(0), a=_on(0), info=_on(1))


def test_one_device_refuses_host_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        pr._one_device(P=_on(0), a=_on(None))


def test_stream_of_another_device_is_refused():
    s = SimpleNamespace(device=torch.device("cuda", 1), cuda_stream=0)
    with pytest.raises(ValueError, match="stream"):
        pr._stream_handle(s, torch.device("cuda", 0))
