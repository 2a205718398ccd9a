"""Host-side logic of bench.py's end-to-end leg on CPU, against a fake NVML:
the process is narrowed to the CPUs that NVML reports nearest the GPU (its
64-bit affinity words decoded bit by bit, intersected with the CPUs the
process may use), the previous CPU set is returned for the restore, and
nothing is changed when NVML is missing, fails, or reports no narrower set."""
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _Props:
    pci_domain_id, pci_bus_id, pci_device_id = 0, 0x1B, 0


def _fake_nvml(words, calls, fail=False):
    m = types.ModuleType("pynvml")
    m.nvmlInit = lambda: calls.append("init")
    m.nvmlShutdown = lambda: calls.append("shutdown")

    def by_bus(bus):
        calls.append(("bus", bus))
        if fail:
            raise RuntimeError("no device")
        return "handle"
    m.nvmlDeviceGetHandleByPciBusId = by_bus
    m.nvmlDeviceGetCpuAffinity = lambda h, n: list(words)[:n]
    return m


@pytest.fixture
def fake_host(monkeypatch):
    state = {"allowed": set(range(128)), "set": []}
    monkeypatch.setattr(os, "sched_getaffinity", lambda pid: set(state["allowed"]))
    monkeypatch.setattr(os, "sched_setaffinity", lambda pid, cpus: state["set"].append(set(cpus)))
    monkeypatch.setattr(os, "cpu_count", lambda: 128)
    import torch
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: _Props())
    return state


def test_binds_to_the_gpu_near_cpus(monkeypatch, fake_host):
    calls = []
    # CPUs 8..15 of word 0 and 64..71 of word 1
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([0xFF00, 0xFF], calls))
    before, desc = bench.bind_host_to_gpu(0)
    near = set(range(8, 16)) | set(range(64, 72))
    assert fake_host["set"] == [near]
    assert before == set(range(128))
    assert desc.startswith("16 of 128 cpus")
    assert ("bus", "00000000:1b:00.0") in calls and calls[-1] == "shutdown"


def test_stays_within_the_allowed_cpus(monkeypatch, fake_host):
    fake_host["allowed"] = set(range(0, 12))
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([0xFF00, 0xFF], []))
    before, desc = bench.bind_host_to_gpu(0)
    assert fake_host["set"] == [set(range(8, 12))] and before == set(range(12))


@pytest.mark.parametrize("words,allowed", [([0xFFFF], set(range(16))),   # nothing narrower
                                           ([0x0F0000], set(range(16))),  # no near CPU allowed
                                           ([0], set(range(16)))])
def test_unchanged_when_not_narrower(monkeypatch, fake_host, words, allowed):
    fake_host["allowed"] = allowed
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(words, []))
    assert bench.bind_host_to_gpu(0) == (None, None)
    assert fake_host["set"] == []


def test_unchanged_when_nvml_fails(monkeypatch, fake_host):
    calls = []
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([0xFF], calls, fail=True))
    assert bench.bind_host_to_gpu(0) == (None, None)
    assert fake_host["set"] == [] and calls[-1] == "shutdown"
