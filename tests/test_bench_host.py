"""Host-side logic of bench.py that needs no GPU: the clock sampler (run
against a fake NVML module in the child process it starts), the rule that
keeps a committed DRAM-traffic figure only while its kernel's sources are
unchanged, the oracle reference arm's JSON line, the multi-GPU launch
(re-execution under torchrun, world-size check), and the weight copies the
small-M back-to-back timing rotates over."""
import sys
import time

import pytest

FAKE_NVML = '''
NVML_CLOCK_SM = 1
_n = [0]
def nvmlInit():
    pass
def nvmlDeviceGetHandleByPciBusId(bus):
    assert bus == "00000000:1B:00.0", bus
    return "h"
def nvmlDeviceGetMaxClockInfo(h, kind):
    return 1965
def nvmlDeviceGetClockInfo(h, kind):
    _n[0] += 1
    return 1900 if _n[0] % 2 else 1800
def nvmlDeviceGetCurrentClocksEventReasons(h):
    return 0x4 | 0x1
'''


def test_clock_sampler_reads_clocks_and_reasons(tmp_path, monkeypatch):
    (tmp_path / "pynvml.py").write_text(FAKE_NVML)
    monkeypatch.setenv("PYTHONPATH", str(tmp_path))
    import bench

    c = bench.ClockSampler(0)
    monkeypatch.setattr(c, "_bus_id", lambda: "00000000:1B:00.0")
    c.start()
    assert c.poller is not None
    time.sleep(0.05)
    out = c.stop()
    assert out["source"] == "nvml"
    assert out["sm_max_mhz"] == 1965
    assert out["sm_mhz"] in (1800, 1900)
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] >= 5


def test_clock_sampler_without_nvml_returns_none(tmp_path, monkeypatch):
    (tmp_path / "pynvml.py").write_text("def nvmlInit():\n    raise RuntimeError('no driver')\n")
    monkeypatch.setenv("PYTHONPATH", str(tmp_path))
    monkeypatch.setenv("PATH", str(tmp_path))  # no nvidia-smi either
    import bench

    c = bench.ClockSampler(0)
    monkeypatch.setattr(c, "_bus_id", lambda: "00000000:1B:00.0")
    c.start()
    assert c.poller is None
    assert c.stop() is None


def test_traffic_entry_goes_null_when_the_kernel_source_changes(tmp_path, monkeypatch):
    """The committed DRAM bytes of a kernel are reported only while the
    hashed sources are the ones the ncu capture was taken of."""
    import hashlib
    import json

    import bench

    csrc = tmp_path / "bit_quantized_lora_quantize_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text("kernel v1")
    (csrc / "h.cuh").write_text("header")
    digest = hashlib.sha256(b"kernel v1" + b"header").hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"gemm": {"sources": ["k.cu", "h.cuh"], "dram_bytes_per_launch": 123, "sources_sha256_16": digest}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_for("gemm") == 123
    assert bench.traffic_for("other") is None
    (csrc / "k.cu").write_text("kernel v2")
    assert bench.traffic_for("gemm") is None


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the oracle on the host cores and
    prints one JSON line with the keys of the bench contract."""
    import json
    import pathlib
    import subprocess

    root = pathlib.Path(__file__).resolve().parents[1]
    out = subprocess.run([sys.executable, str(root / "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], cwd=root, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads(out.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["tokens_per_s"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "llama65b_block_linears"
    import os
    assert d["cpu_baseline"]["cores"] == len(os.sched_getaffinity(0))


def test_multi_gpu_launch_re_execs_under_torchrun():
    """`bench.py --gpus N` without torchrun re-launches itself with one
    process per GPU; under torchrun a world size other than N is an error."""
    import bench

    cmd = bench.torchrun_argv(["--gpus", "2", "--steps", "3"], 2, 29511)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=2" in cmd and "--master-addr=127.0.0.1" in cmd and "--master-port=29511" in cmd
    assert cmd[-3:] == ["--gpus", "2", "--steps", "3"][-3:] and cmd[-4] == "--gpus"
    assert cmd.index(bench.__file__.replace(".pyc", ".py")) < cmd.index("--gpus")


def test_world_size_must_match_gpus(monkeypatch):
    import bench

    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "0")
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "4"])


def test_back_to_back_weight_copies_exceed_three_l2():
    """The small-M back-to-back timing rotates over clones of one packed
    weight: at least four, together at least three times the L2 size, each
    in its own storage with the same contents."""
    import torch

    import bench
    from bit_quantized_lora_quantize_b200.qlora import PackedNF4, packed_sizes

    l2 = 126 << 20
    for N in (8192, 22016):
        numel = N * 8192
        nc, nb, ng = packed_sizes(numel)
        Wp = PackedNF4(torch.randint(0, 256, (nc,), dtype=torch.uint8), torch.randint(0, 256, (nb,), dtype=torch.uint8),
                       torch.rand(ng), (N, 8192))
        nbytes = bench.nf4_bytes(numel)
        assert nbytes == nc + nb + 4 * ng
        ws = bench.weight_copies(Wp, nbytes, l2)
        assert len(ws) >= 4 and len(ws) * nbytes >= 3 * l2
        assert len(ws) == 4 or (len(ws) - 1) * nbytes < 3 * l2  # no more copies than needed
        assert ws[0] is Wp
        ptrs = {w.codes.data_ptr() for w in ws} | {w.absmax_q.data_ptr() for w in ws} | \
               {w.absmax_scale.data_ptr() for w in ws}
        assert len(ptrs) == 3 * len(ws)
        for w in ws[1:]:
            assert torch.equal(w.codes, Wp.codes) and torch.equal(w.absmax_q, Wp.absmax_q)
            assert torch.equal(w.absmax_scale, Wp.absmax_scale)
            assert (w.shape, w.code, w.dq) == (Wp.shape, Wp.code, Wp.dq)
    assert len(bench.weight_copies(Wp, bench.nf4_bytes(8192 * 8192), l2)) == 12
    assert len(bench.weight_copies(Wp, bench.nf4_bytes(22016 * 8192), l2)) == 5
