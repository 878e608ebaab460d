"""The benchmark's roofline accounting without a GPU: the algorithmic bytes and tensor FLOPs it
divides by are the hand counts of the forward pass (q, k, v in and o out in bf16, beta and r in
fp32 per token-head, S_T and d_T out in fp32 per (sequence, head); k~ not counted), the decode
step's bytes are the state's round trip plus its token data, and the committed launch list that
supplies `traffic` and the kernel shares parses into consistent numbers."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from delta_rule_recurrent_osdn_b200 import inputs as W  # noqa: E402


class Shape:
    """Only the fields the accounting reads (no arrays are drawn)."""

    def __init__(self, B, T, H, Dk, Dv, N, apf, init_state, chunk=64):
        self.B, self.T, self.H, self.Dk, self.Dv, self.N, self.chunk = B, T, H, Dk, Dv, N, chunk
        self.r = object() if apf else None
        self.S0 = object() if init_state else None


def test_forward_bytes_at_the_1p3b_shape():
    # per token-head: (2 * 128 + 2 * 128) values x 2 B + beta 4 B + r 4 B = 1032 B;
    # per (sequence, head): S_T (128 x 128) and d_T (128) in fp32 = 66,048 B
    s = Shape(4, 4096, 16, 128, 128, 4, apf=True, init_state=False)
    assert bench.fwd_algorithmic_bytes(s) == 262144 * 1032 + 64 * 66048 == 274_759_680


def test_forward_bytes_count_initial_state_and_skip_r_without_apf():
    # 340M-layer shape (no APF): 1028 B per token-head; long context passes S_0, d_0 in
    s = Shape(8, 2048, 8, 128, 128, 8, apf=False, init_state=False)
    assert bench.fwd_algorithmic_bytes(s) == 8 * 2048 * 8 * 1028 + 64 * 66048
    s = Shape(1, 65536, 16, 128, 128, 1, apf=True, init_state=True)
    assert bench.fwd_algorithmic_bytes(s) == 65536 * 16 * 1032 + 16 * 2 * 66048


def test_forward_flops_at_the_1p3b_shape():
    # per token-head: 5 chunk-local products of 2 C d_k and 3 state products of 2 d_k d_v
    s = Shape(4, 4096, 16, 128, 128, 4, apf=True, init_state=False)
    assert bench.fwd_flops(s) == 262144 * (5 * 2 * 64 * 128 + 3 * 2 * 128 * 128) == 47_244_640_256


def test_decode_bytes_at_256_sequences_by_16_heads():
    # state read + written (2 x 64 KB), d read + written, q, k, v, o in bf16, beta and r
    per_head = 2 * 128 * 128 * 4 + 2 * 128 * 4 + 4 * 128 * 2 + 8
    assert bench.decode_bytes_per_step(256, 16, 128, 128) == 4096 * per_head == 545_292_288


def test_workload_shapes_match_the_named_configs():
    for name, (B, T, H, apf) in {"1p3b_apf": (4, 4096, 16, True),
                                 "340m": (8, 2048, 8, False)}.items():
        cfg = W.CONFIGS[name]
        assert (cfg["B"], cfg["T"], cfg["H"], cfg["Dk"], cfg["Dv"], cfg["apf"]) == \
            (B, T, H, 128, 128, apf), name


def test_committed_launch_list_is_consistent():
    rec = bench.profile_record("fwd_1p3b_apf")
    if rec is None:
        pytest.skip("the committed launch list was taken on other kernel sources")
    shares = {k: float(v) for k, v in (x.split("=") for x in rec["kernel_shares"].split(";"))}
    assert set(shares) == {"precond_prep_kernel", "precond_chain_kernel", "wy_prep_kernel",
                           "chunk_fwd_tc_kernel"}
    assert abs(sum(shares.values()) - 1.0) < 1e-3
    assert max(shares, key=shares.get) == "chunk_fwd_tc_kernel"
    s = Shape(4, 4096, 16, 128, 128, 4, apf=True, init_state=False)
    ratio = float(rec["dram_bytes_per_step"]) / bench.fwd_algorithmic_bytes(s)
    assert 1.0 < ratio < 5.0  # the traffic is real DRAM bytes of a full step, above the floor
