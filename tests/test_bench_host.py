"""Host-side pieces of bench.py: the algorithmic-byte count behind every GB/s
figure (packed index bits/8 + each codebook once + fp16 scale and bias +
bf16 x and y), against sums worked out by hand, and the decode
configuration the JSON line reports."""
import bench
from synth import WORKLOADS


def test_alg_bytes_70b_gate_by_hand():
    spec = WORKLOADS["llama3_70b_mlp"].layers[0][0]          # 28672 x 8192, d = 8, K = 2^16
    idx = 28672 * (8192 // 8) * 16 // 8                       # 58,720,256
    book = 65536 * 8 * 2                                      # 1,048,576
    affine = 2 * 28672 * 2                                    # scale + bias
    xy = 2 * 8192 + 2 * 28672
    assert bench.alg_bytes(spec, 1) == idx + book + affine + xy == 59_957_248


def test_alg_bytes_405b_gate_by_hand():
    spec = WORKLOADS["llama31_405b"].layers[4][0]             # 53248 x 16384, d = 6, 2^12 + 2^4
    nvec = -(-16384 // 6)                                     # 2731 (a partial last vector)
    idx = 53248 * nvec * (12 + 4) // 8
    book = 4096 * 6 * 2 + 16 * 6 * 2
    affine = 2 * 53248 * 2
    xy = 2 * 16384 + 2 * 53248
    assert bench.alg_bytes(spec, 1) == idx + book + affine + xy == 291_242_176


def test_decode_step_configuration():
    cfg = bench.decode_config()
    assert cfg["batch"] == 1 and cfg["bpw"] == 2.0
    assert cfg["layers"] == ["gate_proj", "up_proj", "down_proj"]
    assert set(cfg["index_order"].values()) == {"tile4"}
    step = sum(bench.alg_bytes(s, 1) for s, _ in WORKLOADS["llama3_70b_mlp"].layers)
    assert abs(step - 179.8e6) < 0.1e6                         # the 179.8 MB the step moves


def test_lut_design_bound_70b_gate_up_by_hand():
    """The table design's floor for gate_proj + up_proj in one launch:
    256 groups of four vectors per layer each stream the 1 MiB book
    (536.9 MB at 31 TB/s = 17.32 us), and 2 x 28672 rows x 1024 vectors x
    3 slices = 176.2 M examinations at 4 instructions, 32 lanes, 4 warp
    instructions per clock on 148 SMs at 1.965 GHz = 18.93 us, longer than
    the 18.59 us HBM read of 119.9 MB at 6451.2 GB/s."""
    specs = [s for s, _ in WORKLOADS["llama3_70b_mlp"].layers[:2]]
    b = bench.lut_design_bound(specs, 6451.2)
    assert b["codebook_l2_bytes"] == 2 * 256 * 65536 * 8 * 2 == 536_870_912
    assert b["slice_examinations"] == 2 * 28672 * 1024 * 3 == 176_160_768
    assert abs(b["table_phase_us"] - 536_870_912 / 31e12 * 1e6) < 1e-9
    issue = 176_160_768 * 4 / 32 / (148 * 4 * 1.965e9) * 1e6
    assert abs(b["lookup_phase_issue_us"] - issue) < 1e-9 and abs(issue - 18.93) < 0.01
    assert abs(b["hbm_us"] - 119_914_496 / 6451.2e9 * 1e6) < 1e-9
    assert abs(b["bound_us"] - (17.32 + 18.93)) < 0.01
    assert abs(b["bound_us_at_24tbs"] - (536_870_912 / 24e12 * 1e6 + issue)) < 1e-9
