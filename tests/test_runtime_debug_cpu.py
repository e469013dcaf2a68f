"""KV8_DEBUG mode of the runtime (CPU: the library's check and decode calls
are replaced by recorders, so only the runtime's host logic runs): with the
variable set, every append, decode and step asks kv8_check_indices about its
indices first and raises instead of launching when any is out of range;
without it, nothing is checked."""
import pytest

torch = pytest.importorskip("torch")


@pytest.fixture()
def rt(monkeypatch):
    from paged_int8_kv_b200 import build
    build.build()
    from paged_int8_kv_b200 import runtime
    calls = []
    verdict = {"bad": (0, 0, 0)}

    def fake_check(bt, cl, mcl, nb, slot_mapping=None, stream=None):
        calls.append(("check", bt is not None, cl is not None, mcl, nb,
                      slot_mapping is not None))
        return verdict["bad"]

    def recorder(name):
        def f(*a, **k):
            calls.append((name,))
            return a[0] if a else None
        return f
    monkeypatch.setattr(runtime.B, "kv8_check_indices", fake_check)
    for name in ("kv8_quantize_append", "kv8_paged_decode_attention_form",
                 "kv8_paged_decode_attention_append"):
        monkeypatch.setattr(runtime.B, name, recorder(name))
    monkeypatch.setattr(runtime.B, "kv8_decode_workspace_bytes", lambda *a: 0)
    cache = runtime.PagedKV8Cache(8, 2, device="cpu", poison=False)
    return runtime, cache, calls, verdict


def _args():
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16)
    bt = torch.zeros((2, 4), dtype=torch.int32)
    cl = torch.tensor([5, 17], dtype=torch.int32)
    kv = torch.zeros((2, 2, 128), dtype=torch.bfloat16)
    return q, bt, cl, kv


def test_no_checks_without_the_variable(rt, monkeypatch):
    runtime, cache, calls, _ = rt
    monkeypatch.delenv("KV8_DEBUG", raising=False)
    q, bt, cl, kv = _args()
    cache.decode(q, bt, cl, 64, chunk_tokens=0)
    cache.append(kv, kv, torch.zeros(2, dtype=torch.int64))
    assert [c[0] for c in calls] == ["kv8_paged_decode_attention_form",
                                     "kv8_quantize_append"]
    monkeypatch.setenv("KV8_DEBUG", "0")
    assert not runtime.debug_checks_enabled()


def test_checks_run_first_and_pass_through(rt, monkeypatch):
    runtime, cache, calls, _ = rt
    monkeypatch.setenv("KV8_DEBUG", "1")
    q, bt, cl, kv = _args()
    cache.decode(q, bt, cl, 64, chunk_tokens=0)
    cache.step(q, kv, kv, bt, cl, 64, chunk_tokens=0)
    cache.append(kv, kv, torch.zeros(2, dtype=torch.int64))
    assert calls == [("check", True, True, 64, 8, False),
                     ("kv8_paged_decode_attention_form",),
                     ("check", True, True, 64, 8, False),
                     ("kv8_paged_decode_attention_append",),
                     ("check", False, False, 0, 8, True),
                     ("kv8_quantize_append",)]


def test_bad_indices_raise_before_launch(rt, monkeypatch):
    runtime, cache, calls, verdict = rt
    monkeypatch.setenv("KV8_DEBUG", "1")
    q, bt, cl, kv = _args()
    verdict["bad"] = (0, 2, 0)
    with pytest.raises(ValueError, match="2 block-table entries"):
        cache.decode(q, bt, cl, 64, chunk_tokens=0)
    verdict["bad"] = (1, 0, 0)
    with pytest.raises(ValueError, match="1 context lengths"):
        cache.step(q, kv, kv, bt, cl, 64, chunk_tokens=0)
    verdict["bad"] = (0, 0, 3)
    with pytest.raises(ValueError, match="3 slots"):
        cache.append(kv, kv, torch.zeros(2, dtype=torch.int64))
    assert all(c[0] == "check" for c in calls)


def test_kivi_runtime_forwards_and_checks(rt, monkeypatch):
    runtime, _, calls, verdict = rt
    seen = []

    def rec(name):
        def f(*a, **k):
            seen.append((name, a, k))
            return a[5] if name == "decode" else None
        return f
    monkeypatch.setattr(runtime.B, "kv8_kivi_append", rec("append"))
    monkeypatch.setattr(runtime.B, "kv8_kivi_paged_decode_attention", rec("decode"))
    c = runtime.PagedKiviCache(8, 2, 2, device="cpu")
    assert c.records.shape == (8, 2, 2176) and c.tail.shape == (2, 2, 2, 16, 128)
    q, bt, cl, kv = _args()
    cu = torch.tensor([0, 1, 2], dtype=torch.int32)
    monkeypatch.delenv("KV8_DEBUG", raising=False)
    c.append(kv, kv, cu, cl, bt, 1)
    out = c.decode(q, bt, cl, 64, chunk_tokens=0, out_dtype=torch.float32)
    assert [s[0] for s in seen] == ["append", "decode"] and not calls
    assert seen[0][1][5] is c.records and seen[0][1][6] is c.tail
    assert seen[1][1][1] is c.records and out.dtype == torch.float32
    monkeypatch.setenv("KV8_DEBUG", "1")
    verdict["bad"] = (0, 1, 0)
    with pytest.raises(ValueError):
        c.decode(q, bt, cl, 64, chunk_tokens=0)
    with pytest.raises(ValueError):
        c.append(kv, kv, cu, cl, bt, 1)
    assert len(seen) == 2


def test_check_indices_needs_something_to_check():
    from paged_int8_kv_b200 import build
    build.build()
    from paged_int8_kv_b200 import _binding
    with pytest.raises(ValueError):
        _binding.kv8_check_indices(None, None, 0, 8)
