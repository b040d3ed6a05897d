"""Host-side pieces of bench.py that need no GPU."""
import os
import sys
from types import SimpleNamespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def test_nvml_bus_id_is_a_string():
    # torch reports the PCI location as integers; NVML takes the
    # "domain:bus:device.function" string (an integer would be read as an address).
    import bench
    props = SimpleNamespace(pci_domain_id=0, pci_bus_id=0x1B, pci_device_id=0)
    bus = bench.ClockSampler.pci_bus_id(props)
    assert isinstance(bus, str)
    assert bus == "0000:1b:00.0"
    with pytest.raises(TypeError):
        bench.ClockSampler.pci_bus_id(SimpleNamespace(pci_domain_id=0, pci_bus_id="1b", pci_device_id=0))


def test_clock_summary_without_sampling_source():
    import bench
    c = bench.ClockSampler(0)
    c.nvml = None
    assert c.summary()["reasons"] == ["clock sampling unavailable"]
