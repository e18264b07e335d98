"""CPU-only checks of bench.py's bookkeeping and of the no-fallback rule."""
import itertools
import os

import pytest
import torch

import bench
import workloads


@pytest.mark.parametrize("causal", [False, True])
def test_visible_pairs_matches_brute_force(causal):
    w = workloads.Workload("t", 0, 3, 2, 37, 64, causal)
    for kv_len in (None, torch.tensor([0, 20, 99], dtype=torch.int32)):
        lims = [37] * 3 if kv_len is None else [min(max(int(x), 0), 37) for x in kv_len]
        brute = sum(1 for b, i, j in itertools.product(range(3), range(37), range(37))
                    if j < lims[b] and (not causal or j <= i)) * w.H
        assert bench.visible_pairs(w, kv_len) == brute


def test_visible_pairs_of_the_workloads():
    w5 = workloads.get(5)
    assert bench.visible_pairs(w5) == w5.H * w5.N * (w5.N + 1) // 2
    assert 4.0 * w5.d * bench.visible_pairs(w5) == pytest.approx(w5.flops(), rel=1e-4)


def test_source_hash_ignores_comments(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_text("int a = 1; // one\n/* block */ int b = 2;\n")
    monkeypatch.setattr(bench, "KERNEL_SOURCES", [str(src)])
    monkeypatch.setattr(bench, "ROOT", "/")
    h1 = bench.kernel_source_hash()
    src.write_text("int a = 1;   // a different comment\n\n/* another */\nint b = 2;\n")
    assert bench.kernel_source_hash() == h1
    src.write_text("int a = 1; int b = 3;\n")
    assert bench.kernel_source_hash() != h1


def test_recorded_traffic_requires_matching_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic_x.txt").write_text(
        "# comment: lines with a colon after a hash are ignored\n"
        "kernel_source_sha256_16: abc\nmeasured_case: B1 H2\n"
        "dram_read_bytes_per_launch: 100\ndram_write_bytes_per_launch: 23\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.recorded_traffic("x") == {"read": 100.0, "write": 23.0, "case": "B1 H2"}
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "def")
    assert bench.recorded_traffic("x") is None


def test_missing_extension_fails_loudly(tmp_path):
    import io_aware_exact_18_b200 as fa
    with pytest.raises(ImportError):
        fa.load_library(os.path.join(str(tmp_path), "libfa.so"))


def _input_bytes(w):
    kv = w.kv_heads
    return 2 * w.B * w.N * w.d * (w.H + 2 * kv)


def test_l2_policy_flushes_the_workloads_that_fit_near_the_l2():
    for idx in (1, 2, 3, 4):
        flush, note = bench.l2_policy(_input_bytes(workloads.get(idx)))
        assert flush and note.startswith("flush:")
    flush, note = bench.l2_policy(_input_bytes(workloads.get(5)))
    assert not flush and note.startswith("no flush:") and "384 MiB" in note
    for dw in workloads.DECODE_WORKLOADS:
        kv_bytes = 2 * 2 * dw.B * dw.H_kv * dw.Nk * dw.d
        assert not bench.l2_policy(kv_bytes)[0]
    assert bench.FLUSH_BYTES > 2 * bench.L2_BYTES
    assert bench.l2_policy(int(1.5 * bench.L2_BYTES))[0] is False
    assert bench.l2_policy(int(1.5 * bench.L2_BYTES) - 1)[0] is True


class _FakeCuda:
    """Stands in for torch.cuda in time_steps: records the order of events,
    steps and flushes, and gives each event pair a fixed duration."""

    def __init__(self, log):
        self.log = log
        cuda = self

        class Event:
            n = 0

            def __init__(self, enable_timing=False):
                assert enable_timing
                Event.n += 1
                self.id = Event.n

            def record(self, stream):
                cuda.log.append(("record", self.id))

            def elapsed_time(self, other):
                return 2.0 * (other.id - self.id)

        self.Event = Event

    class _Ctx:
        def __enter__(self):
            return self

        def __exit__(self, *a):
            return False

    def stream(self, s):
        return self._Ctx()


class _FakeStream:
    def __init__(self, log):
        self.log = log

    def synchronize(self):
        self.log.append(("sync",))


class _FakeBuf:
    def __init__(self, log):
        self.log = log

    def fill_(self, v):
        self.log.append(("flush", v))


def test_time_steps_flushes_before_each_step_and_times_only_the_step():
    log = []
    fake_torch = type("T", (), {})()
    fake_torch.cuda = _FakeCuda(log)
    step = lambda: log.append(("step",))  # noqa: E731
    ms = bench.time_steps(fake_torch, _FakeStream(log), step, 3, _FakeBuf(log))
    kinds = [e[0] for e in log]
    assert kinds == ["flush", "record", "step", "record"] * 3 + ["sync"]
    assert ms == pytest.approx(2.0)   # each pair is consecutive events: 2.0 ms apiece

    log.clear()
    ms = bench.time_steps(fake_torch, _FakeStream(log), step, 4, None)
    assert [e[0] for e in log] == ["record"] + ["step"] * 4 + ["record", "sync"]
    assert ms == pytest.approx(2.0 / 4)


def test_decode_kernel_name_follows_the_dispatch_rule():
    """The decode line names the transposed tile exactly where the library
    takes it (d = 128, query heads per K/V head x query rows <= 8), and the
    merge only when there is more than one key range."""
    import workloads
    w1, w2 = workloads.DECODE_WORKLOADS[0], workloads.DECODE_WORKLOADS[1]
    assert bench.decode_kernel_name(w1, 1) == "fa_decode_sm100<128,bf16>"
    assert bench.decode_kernel_name(w2, 16) == \
        "fa_decode_sm100<128,bf16> + fa_splitkv_combine<128>"
    wide = workloads.DecodeWorkload("wide", 1, 32, 2, 1, 4096, 128)   # 16 heads per K/V head
    assert bench.decode_kernel_name(wide, 4).startswith("fa_fwd_sm100<128,1,general>")
    d64 = workloads.DecodeWorkload("d64", 1, 32, 8, 1, 4096, 64)
    assert bench.decode_kernel_name(d64, 1) == "fa_fwd_sm100<64,1,general>"
