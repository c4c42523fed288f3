"""CPU checks of how bench.py finds the GPU whose clocks it samples, against a
fake NVML: NVML numbers every GPU of the machine and ignores
CUDA_VISIBLE_DEVICES, so the CUDA device is matched by its PCI location."""
from types import SimpleNamespace

import bench


class FakeNVML:
    def __init__(self, pci, forbidden=()):
        self.pci = pci                      # NVML index -> (domain, bus, device)
        self.forbidden = set(forbidden)     # indices that raise, as for a GPU of another container

    def nvmlDeviceGetCount(self):
        return len(self.pci)

    def nvmlDeviceGetHandleByIndex(self, i):
        if i in self.forbidden:
            raise RuntimeError("no permission")
        return ("handle", i)

    def nvmlDeviceGetPciInfo(self, h):
        d, b, v = self.pci[h[1]]
        return SimpleNamespace(domain=d, bus=b, device=v)


def props(domain, bus, device):
    return SimpleNamespace(pci_domain_id=domain, pci_bus_id=bus, pci_device_id=device)


MACHINE = [(0, 0x18, 0), (0, 0x2A, 0), (0, 0x3A, 0), (0, 0x5D, 0),
           (0, 0x9A, 0), (0, 0xAB, 0), (0, 0xBA, 0), (0, 0xDB, 0)]


def test_visible_device_is_found_by_pci_location():
    # CUDA_VISIBLE_DEVICES=5: CUDA device 0 is the machine's sixth GPU
    assert bench.nvml_handle_of(FakeNVML(MACHINE), props(0, 0xAB, 0), 0) == ("handle", 5)


def test_gpus_that_cannot_be_queried_are_skipped():
    assert bench.nvml_handle_of(FakeNVML(MACHINE, forbidden={0, 1, 2}), props(0, 0xBA, 0), 0) == ("handle", 6)


def test_index_is_the_fallback():
    nv = FakeNVML(MACHINE)
    assert bench.nvml_handle_of(nv, None, 3) == ("handle", 3)                  # no CUDA properties
    assert bench.nvml_handle_of(nv, props(1, 0x18, 0), 2) == ("handle", 2)     # no GPU at that location


def test_sampler_samples_the_matched_gpu(monkeypatch):
    """ClockSampler end to end on the fake: the handle, the maximum clock and
    the samples (with throttle reasons) all come from the GPU at the CUDA
    device's PCI location."""
    import sys
    import time
    import torch

    class Fake(FakeNVML):
        NVML_CLOCK_SM = 1

        def nvmlInit(self):
            pass

        def nvmlDeviceGetMaxClockInfo(self, h, kind):
            return 1965 if h == ("handle", 5) else 1000

        def nvmlDeviceGetClockInfo(self, h, kind):
            return 1965 if h == ("handle", 5) else 500

        def nvmlDeviceGetCurrentClocksEventReasons(self, h):
            return 0x4 if h == ("handle", 5) else 0x40

    monkeypatch.setitem(sys.modules, "pynvml", Fake(MACHINE))
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: props(0, 0xAB, 0))
    s = bench.ClockSampler(0)
    assert s.h == ("handle", 5) and s.max_mhz == 1965
    with s:
        time.sleep(0.01)
    assert s.samples and set(s.samples) == {1965}
    assert s.reasons == {"sw_power_cap"}
