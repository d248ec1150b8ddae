"""Host logic of the sequence-parallel prefill on CPU: the order of one rank's
calls (local state, one gather, prefix, prefill from that state) and the
arguments they pass, with the library calls replaced by recorders."""
import pytest
import torch

from long_context_02_b200 import sp


@pytest.fixture
def calls(monkeypatch):
    log = []
    L = sp.L
    monkeypatch.setattr(L, "workspace", lambda *a, **k: torch.zeros(16, dtype=torch.uint8))
    monkeypatch.setattr(L, "la_prefill_state",
                        lambda k, v, s, s_in, out, ws, stream=None: log.append(
                            ("state", tuple(k.shape), s_in is None)) or out.fill_(1.0))
    monkeypatch.setattr(L, "la_state_prefix",
                        lambda states, s, lens, r, out, stream=None: log.append(
                            ("prefix", tuple(states.shape), list(lens), r)) or out.fill_(2.0))
    monkeypatch.setattr(L, "la_prefill_with_state",
                        lambda q, k, v, s, s_in, o, st, ws, stream=None: log.append(
                            ("prefill", tuple(q.shape), float(s_in.mean()))))
    return log


def test_one_rank_makes_its_calls_in_order(calls):
    B, H, n, d, R, rank = 1, 2, 5, 8, 3, 1
    q = torch.zeros((B, H, n, d))
    gathered = []

    def gather(s_loc):
        gathered.append(s_loc.clone())
        return torch.stack([s_loc] * R)

    sp.sp_prefill(q, q, q, None, [4, n, 7], rank, q.clone(), None, gather)
    assert [c[0] for c in calls] == ["state", "prefix", "prefill"]
    assert calls[0] == ("state", (B, H, n, d), True)          # the chunk alone, from zero
    assert len(gathered) == 1 and torch.all(gathered[0] == 1.0)
    assert calls[1] == ("prefix", (R, B, H, d, d), [4, n, 7], rank)
    assert calls[2] == ("prefill", (B, H, n, d), 2.0)          # continued from the prefix


def test_chunk_length_must_match(calls):
    q = torch.zeros((1, 2, 5, 8))
    with pytest.raises(ValueError):
        sp.sp_prefill(q, q, q, None, [5, 6], 1, q, None, lambda s: s)
    assert calls == []
