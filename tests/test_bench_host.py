"""Host-side pieces of bench.py (CPU): FLOP definitions, the DRAM-traffic records
and their source hashes, and the argument surface of the timed passes."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import bench as b
    return b


def test_flop_definitions(bench):
    import synth
    c = synth.CONFIGS["hunyuan108k"]
    info = {"block_pairs": 1000, "kept_pairs": 600}
    d, BH = c["d"], c["B"] * c["H"]
    assert bench.flops_per_call(info, c, "block") == 4 * d * 1000 * BH
    assert bench.flops_per_call(info, c, "token_exact") == 4 * d * 600 * BH
    # the backward counts the five products S, dP, dQ, dK, dV: 2.5 times the forward
    assert bench.flops_per_call(info, c, "block", "bwd") == 2.5 * bench.flops_per_call(info, c, "block")


def test_traffic_records_follow_the_kernel_sources(bench, tmp_path, monkeypatch):
    # the committed records parse, and each names the hash of its own kernel's sources
    for kind in ("fwd", "bwd"):
        path = os.path.join(ROOT, "profiles", f"attn_{kind}_traffic.txt")
        assert os.path.exists(path), path
        for rel in bench.ATTN_SOURCES[kind]:
            assert os.path.exists(os.path.join(ROOT, rel)), rel
    assert bench.recorded_traffic("no_such_workload", "block", "radial") is None
    # a record taken on other sources is not reported
    fake_root = tmp_path
    (fake_root / "profiles").mkdir()
    (fake_root / "profiles" / "attn_fwd_traffic.txt").write_text(
        "hunyuan108k/radial/block sources=0000000000000000 dram_bytes_per_launch=123\n")
    for rel in bench.ATTN_SOURCES["fwd"]:
        dst = fake_root / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        dst.write_bytes(open(os.path.join(ROOT, rel), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    assert bench.recorded_traffic("hunyuan108k", "block", "radial") is None
    good = bench.sources_sha256("fwd")
    (fake_root / "profiles" / "attn_fwd_traffic.txt").write_text(
        f"hunyuan108k/radial/block sources={good} dram_bytes_per_launch=123\n")
    assert bench.recorded_traffic("hunyuan108k", "block", "radial") == 123


def test_workload_description_names_the_mask(bench):
    import synth
    c = synth.CONFIGS["hunyuan108k"]
    text = bench.workload_desc("hunyuan108k", c["masks"][2], "block", c)
    assert "3600 global (sink) tokens" in text and "n=108000" in text
    w = synth.CONFIGS["wan_radial"]
    assert "W=16" in bench.workload_desc("wan_radial", w["masks"][1], "block", w)


def test_pass_choices(bench, monkeypatch):
    for argv, want in ([["bench.py"], "fwd"], [["bench.py", "--pass", "bwd"], "bwd"],
                       [["bench.py", "--pass", "stream", "--workload", "wan_radial", "--mask", "1"], "stream"],
                       [["bench.py", "--pass", "policy"], "policy"]):
        monkeypatch.setattr(sys, "argv", argv)
        args = bench.parse_args()
        assert args.pass_ == want
        assert args.steps >= 1 and args.warmup >= 3


def _reference_line(args, rank="0"):
    import json
    import subprocess
    env = dict(os.environ, RANK=rank)
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", *args], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = out.stdout.strip().splitlines()
    return json.loads(lines[-1]) if lines else None


@pytest.mark.parametrize("args", [["--workload", "tiny_radial", "--steps", "1", "--warmup", "3"],
                                  ["--pass", "stream", "--workload", "wan_radial", "--mask", "1",
                                   "--steps", "1", "--warmup", "3"]], ids=["fwd_tiny", "stream_wan"])
def test_reference_arm_line(args):
    """The reference arm (the oracle on the host cores) prints one line with the
    contract's keys; a rank other than 0 prints nothing and exits 0."""
    line = _reference_line(args)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert _reference_line(args, rank="1") is None


def test_forward_kernel_name_follows_the_library_choice(bench):
    """Rows of >= 4096 computed keys on average keep bf16 P; fewer keep hi + lo P."""
    import synth
    big = synth.CONFIGS["hunyuan108k"]
    info = {"block_pairs": 321300 * 128 * 128, "kept_pairs": 4547300400}
    assert bench.fwd_kernel_name(info, big, "block") == "attn_fwd_kernel<128, false>"
    tiny = synth.CONFIGS["tiny_radial"]
    assert bench.fwd_kernel_name({"block_pairs": 512 * 512, "kept_pairs": 191872}, tiny, "token_exact") == \
        "attn_fwd_kernel<64, true>"


def test_traffic_record_key_tells_sink_masks_apart(bench):
    """A mask with global tokens walks other tiles: it does not take the record of
    the plain mask of the same family."""
    assert bench.mask_key({"family": "radial"}) == "radial"
    assert bench.mask_key({"family": "radial", "sink_tokens": 3600}) == "radial+sink3600"
    plain = bench.recorded_traffic("hunyuan108k", "block", "radial")
    sink = bench.recorded_traffic("hunyuan108k", "block", "radial+sink3600")
    assert sink is None or sink != plain
    assert bench.recorded_traffic("hunyuan108k", "block", "radial+sink1") is None
