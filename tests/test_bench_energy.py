"""The bench's energy meter against a stand-in NVML (CPU only): it reads the total-energy
counter before and after the timed region, reports joules per token, finds the GPU by
PCI bus id, degrades to no figure when NVML fails, and never calls a setter or a reset."""
import bench


class FakeNvml:
    def __init__(self, readings, bus_ok=True, fail_init=False):
        self.readings = list(readings)
        self.bus_ok, self.fail_init = bus_ok, fail_init
        self.calls = []

    def __getattr__(self, name):
        if name.startswith("nvmlDeviceSet") or name.startswith("nvmlDeviceReset") or "Clock" in name:
            raise AssertionError(f"meter touched {name}")
        raise AttributeError(name)

    def nvmlInit(self):
        self.calls.append("init")
        if self.fail_init:
            raise RuntimeError("no driver")

    def nvmlShutdown(self):
        self.calls.append("shutdown")

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        self.calls.append(("bus", bus))
        if not self.bus_ok:
            raise RuntimeError("not found")
        return ("h", bus)

    def nvmlDeviceGetHandleByIndex(self, i):
        self.calls.append(("index", i))
        return ("h", i)

    def nvmlDeviceGetTotalEnergyConsumption(self, h):
        self.calls.append(("energy", h))
        return self.readings.pop(0)


def test_energy_per_token_from_two_counter_readings():
    nv = FakeNvml([5_000_000, 5_250_000])            # millijoules
    with bench.EnergyMeter(0, "00000000:1B:00.0", nvml=nv) as em:
        em.start()
        em.stop()
    s = em.summary(tokens=500)
    assert abs(s["joules"] - 250.0) < 1e-9
    assert abs(s["j_per_token"] - 0.5) < 1e-12
    assert abs(s["tokens_per_j"] - 2.0) < 1e-12
    assert ("bus", "00000000:1B:00.0") in nv.calls and not any(c[0] == "index" for c in nv.calls if isinstance(c, tuple))
    assert nv.calls[-1] == "shutdown"


def test_falls_back_to_index_when_bus_id_unknown():
    nv = FakeNvml([10, 20], bus_ok=False)
    with bench.EnergyMeter(3, "bad", nvml=nv) as em:
        em.start()
        em.stop()
    assert ("index", 3) in nv.calls
    assert em.summary(tokens=1)["joules"] == 0.01


def test_no_figure_when_nvml_unavailable_or_counter_wraps():
    nv = FakeNvml([], fail_init=True)
    with bench.EnergyMeter(0, None, nvml=nv) as em:
        em.start()
        em.stop()
    assert em.summary(tokens=10) is None
    nv = FakeNvml([200, 100])                        # counter went backwards (driver reload)
    with bench.EnergyMeter(0, None, nvml=nv) as em:
        em.start()
        em.stop()
    assert em.summary(tokens=10) is None
