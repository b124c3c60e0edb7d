"""The roofline's measured-traffic records are keyed on a kernel's device code: the source file
up to the closing brace of the kernel's definition.  Host code after it may change; anything
before it (constants, helpers, the kernel) invalidates the record."""
import importlib.util
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


SRC = """constexpr int kTile = 64;
__device__ int helper(int x) { return x + kTile; }
__global__ void
my_kernel(int *p)
{
    p[0] = helper(1);
}

bool host_helper() { return true; }
"""
DEF = "\nmy_kernel(int *p)\n"


def test_host_code_after_the_kernel_does_not_change_the_key():
    b = load_bench()
    assert b.device_code_sha(SRC, DEF) == b.device_code_sha(SRC + "int more_host_code();\n", DEF)
    assert b.device_code_sha(SRC, DEF) == b.device_code_sha(SRC.replace("return true", "return false"), DEF)


def test_device_code_changes_the_key():
    b = load_bench()
    base = b.device_code_sha(SRC, DEF)
    assert b.device_code_sha(SRC.replace("kTile = 64", "kTile = 32"), DEF) != base
    assert b.device_code_sha(SRC.replace("helper(1)", "helper(2)"), DEF) != base


def test_committed_records_name_a_kernel_definition_present_in_their_file():
    import json
    d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for name, e in d.items():
        if name.startswith("_"):
            continue
        # a record for one kernel is named for its file; one for a call of several kernels
        # lists them
        kernels = e["kernels"] if "kernels" in e else [dict(e, file=name)]
        for k in kernels:
            text = open(os.path.join(ROOT, "gated_delta_rule_78_b200", "csrc", k["file"])).read()
            assert k["kernel_def"] in text, (name, k["file"])
        assert e.get("bytes_per_launch", e.get("bytes_per_call", 0)) > 0


def test_a_record_over_several_kernels_needs_all_of_them_unchanged(tmp_path, monkeypatch):
    import json
    b = load_bench()
    csrc = tmp_path / "gated_delta_rule_78_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    (csrc / "a.cu").write_text(SRC)
    (csrc / "b.cu").write_text(SRC.replace("my_kernel", "other_kernel"))
    rec = {"bytes_per_call": 123, "kernels": [
        {"file": "a.cu", "kernel_def": DEF, "sha256_device": b.device_code_sha(SRC, DEF)},
        {"file": "b.cu", "kernel_def": "\nother_kernel(int *p)\n",
         "sha256_device": b.device_code_sha(SRC.replace("my_kernel", "other_kernel"), "\nother_kernel(int *p)\n")}]}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"call": rec}))
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    assert b.kernel_traffic("call") == 123
    (csrc / "b.cu").write_text(SRC.replace("my_kernel", "other_kernel").replace("kTile = 64", "kTile = 32"))
    assert b.kernel_traffic("call") is None
