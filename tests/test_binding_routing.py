"""Host logic of the binding that needs no GPU: forward_2to8 sends calls of
more than one token to the 2:4 forward when it is given the 2:4 packing of
the same matrix (a 2:8 pattern is a 2:4 pattern), and keeps single tokens,
or calls without that packing, on the 2:8 entry point."""
import torch

import sparse_rank_linear_02_b200 as slr


class _Lib:
    def __init__(self):
        self.calls = []

    def slr_forward_2to8(self, *args):
        self.calls.append("slr_forward_2to8")
        return 0


def _tensors(M, d_in=64, d_out=16, r=8):
    X = torch.zeros((M, d_in), dtype=torch.bfloat16)
    v8 = torch.zeros((d_out, d_in // 4), dtype=torch.bfloat16)
    m8 = torch.zeros((d_out, d_in // 8), dtype=torch.uint8)
    v4 = torch.zeros((d_out, d_in // 2), dtype=torch.bfloat16)
    m4 = torch.zeros((d_out, d_in // 8), dtype=torch.uint8)
    U = torch.zeros((d_out, r), dtype=torch.bfloat16)
    V = torch.zeros((r, d_in), dtype=torch.bfloat16)
    return X, v8, m8, v4, m4, U, V


def test_forward_2to8_routing(monkeypatch):
    fake = _Lib()
    routed = []
    monkeypatch.setattr(slr, "_lib", fake)
    monkeypatch.setattr(slr, "_stream", lambda: None)
    monkeypatch.setattr(slr, "workspace_size", lambda *a: 0)
    monkeypatch.setattr(slr, "forward", lambda X, vals, meta, U, V, out=None, workspace=None:
                        routed.append((X.shape[0], vals.shape[1])) or "2:4")
    for M in (2, 4, 300):
        X, v8, m8, v4, m4, U, V = _tensors(M)
        assert slr.forward_2to8(X, v8, m8, U, V, vals4=v4, meta4=m4) == "2:4"
        assert routed[-1] == (M, v4.shape[1])          # the 2:4 packing, not the 2:8 one
    n = len(routed)
    X, v8, m8, v4, m4, U, V = _tensors(1)               # one token: the 2:8 kernel
    slr.forward_2to8(X, v8, m8, U, V, vals4=v4, meta4=m4)
    X, v8, m8, v4, m4, U, V = _tensors(16)              # no 2:4 packing given: the 2:8 kernel
    slr.forward_2to8(X, v8, m8, U, V)
    assert len(routed) == n
    assert fake.calls == ["slr_forward_2to8", "slr_forward_2to8"]
