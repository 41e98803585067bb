"""CPU checks of bench.py's byte model and bookkeeping (no GPU): the
algorithmic bytes follow the effective-bit formula, the per-kernel split adds
up, the stacks exceed L2 as stated, and a traffic record is used only for the
kernel source it was captured on."""
import hashlib
import json
import os
from fractions import Fraction

import pytest

import bench
from oracle import littlebit_oracle as orc

SHAPES = [(4096, 4096, 86, True), (4096, 4096, 188, False), (8192, 28672, 620, False),
          (28672, 8192, 302, True), (4096, 11008, 133, True), (512, 512, 32, False)]


@pytest.mark.parametrize("a,b,s,res", SHAPES)
def test_weight_bytes_are_the_effective_bit_count(a, b, s, res):
    """With no activations, the bytes per matrix are exactly eff_bit * a * b / 8
    (the LittleBit-2 column's formula: signs, plus 16-bit h, g and l)."""
    weight_bytes = Fraction(bench.algorithmic_bytes(a, b, s, res, 0)).limit_denominator(8)
    assert weight_bytes * 8 == orc.eff_bits_exact(a, b, s, res) * a * b


@pytest.mark.parametrize("a,b,s,res", SHAPES)
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_kernel_split_adds_up(a, b, s, res, batch):
    kb = bench.kernel_bytes(a, b, s, res, batch)
    assert set(kb) == set(bench.KERNELS)
    assert sum(kb.values()) == pytest.approx(bench.algorithmic_bytes(a, b, s, res, batch), rel=1e-12)
    # activations: x is read by the quantise pass, y written by the output pass
    assert kb["quantise"] - bench.kernel_bytes(a, b, s, res, 0)["quantise"] == 2 * batch * a
    assert kb["output_pass"] - bench.kernel_bytes(a, b, s, res, 0)["output_pass"] == 2 * batch * b


def test_worked_example_7b_attention_residual():
    # 2 paths x (86*8192/8 sign bytes + 2*(8192 + 86) scale bytes) + 2*8192 activation bytes
    assert bench.algorithmic_bytes(4096, 4096, 86, True, 1) == 2 * (88064 + 16556) + 16384


@pytest.mark.parametrize("name", sorted(bench.WORKLOADS))
def test_stacks_exceed_l2(name):
    l2 = 126 * 2 ** 20
    mats = bench.WORKLOADS[name]["mats"]
    model_layers = bench.WORKLOADS[name].get("model_layers", 1)
    reps = bench.stack_reps_for_l2(mats, 1, l2, 4.0, model_layers)
    per = sum(bench.algorithmic_bytes(*m, 1) for m in mats)
    assert reps * per >= 4 * l2
    # the model's own depth, or the fewest copies that reach 4x L2
    assert reps == model_layers or (reps - 1) * per < 4 * l2


def test_headline_is_the_70b_mlp_stack():
    """The default (headline) workload is the 80-layer Llama-2-70B MLP stack at
    0.1 BPW, whose packed bytes are several times the L2 cache."""
    wl = bench.WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert wl["mats"] == [(8192, 28672, 620, False), (8192, 28672, 620, False), (28672, 8192, 620, False)]
    assert wl["model_layers"] == 80
    per = sum(bench.algorithmic_bytes(*m, 1) for m in wl["mats"])
    assert 80 * per > 5 * 126 * 2 ** 20


def test_traffic_record_only_for_the_captured_source(tmp_path, monkeypatch):
    csrc = tmp_path / "latent_binary_factorization_b200" / "csrc"
    csrc.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = b"// kernel source\n"
    (csrc / "decode.cu").write_bytes(src)
    digest = hashlib.sha256(src).hexdigest()[:16]
    rec = {"w": {"output_pass": {"decode_cu_sha256_16": digest, "dram_bytes_per_model_layer": 1000.5}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("output_pass", "w", 10) == 10005
    assert bench.traffic_record("latent_pass", "w", 10) is None
    assert bench.traffic_record("output_pass", "other", 10) is None
    (csrc / "decode.cu").write_bytes(src + b"// changed\n")
    assert bench.traffic_record("output_pass", "w", 10) is None


def test_committed_traffic_records_name_a_source_hash():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    assert rec
    for workload, kernels in rec.items():
        if not isinstance(kernels, dict):
            continue
        for kernel, r in kernels.items():
            if isinstance(r, dict) and "dram_bytes_per_model_layer" in r:
                assert len(r["decode_cu_sha256_16"]) == 16, (workload, kernel)


def test_shared_inputs_are_read_once_in_the_byte_model():
    """The 7B full layer's q, k, v share one input and gate, up another: the
    model layer's bytes count each shared input once."""
    wl = bench.WORKLOADS["7b_layer_0.1bpw_residual"]
    full = sum(bench.algorithmic_bytes(*m, 1) for m in wl["mats"])
    saved = bench.shared_x_bytes(wl["mats"], wl["x_groups"], 1)
    assert saved == 2 * (2 * 4096) + 1 * (2 * 4096)     # two extra reads for q,k,v; one for gate,up
    assert bench.layer_bytes("7b_layer_0.1bpw_residual", 1) == full - saved
    assert bench.shared_x_bytes([(4096, 4096, 86, True)], None, 1) == 0
