"""bench.py's default run attaches short runs of the other workloads; a run
that fails (here: no GPU in the process) becomes an error entry and never
takes the headline line down.  Runs on the CPU."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_secondary_only_on_the_default_single_process_run(monkeypatch):
    b = _bench()
    for k in ("TORCHELASTIC_RUN_ID", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    monkeypatch.setattr("sys.argv", ["bench.py"])
    assert b.wants_secondary(b.parse())
    for extra in (["--no-secondary"], ["--workload", "robertson"], ["--dtype", "f32"], ["--n", "4096"],
                  ["--impl", "reference"]):
        monkeypatch.setattr("sys.argv", ["bench.py", *extra])
        assert not b.wants_secondary(b.parse()), extra
    monkeypatch.setattr("sys.argv", ["bench.py"])
    monkeypatch.setenv("TORCHELASTIC_RUN_ID", "x")
    assert not b.wants_secondary(b.parse())


def test_failed_secondary_is_an_error_entry(monkeypatch):
    b = _bench()
    monkeypatch.setattr(b, "SECONDARY", [("robertson_ros2", ["--workload", "robertson"], 0),
                                         ("bad", ["--workload", "no_such_workload"], 0)])
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "")
    res = b.run_secondary()
    assert set(res) == {"robertson_ros2", "bad"}
    assert all("error" in v and v["error"].startswith("exit ") for v in res.values()), res
