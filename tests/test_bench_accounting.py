"""The algorithmic work bench.py divides by (host only, no GPU).

The roofline fractions on the bench line are algorithmic bytes (or flops) over
a measured time, so the counts themselves need a pin that is not the formula
retyped:
- bytes: the tensors one call actually reads and writes, built by the same
  seeded generator the bench uses, summed by their own nbytes;
- flops: an explicit enumeration of the multiply-adds of the causal chunked
  form ("Mamba2" knowledge page, the two-stage chunk scan: C.B^T on j <= i
  once per group, the weighted C.B^T.x on j <= i, the chunk state B^T(w x)
  and the output C.h per head), counted one (i, j) pair at a time.
"""
import math

import pytest
import torch

import bench
from state_space_sequence_scan_b200.inputs import SCAN_CONFIGS, STEP_CONFIGS, make_scan_inputs, make_step_inputs


def _scan_tensor_bytes(cfg):
    """Bytes of every input tensor of one call plus its outputs: y [b,L,H,P]
    fp32 and final_state [b,H,N,P] fp32."""
    inp = make_scan_inputs(cfg)
    total = sum(t.numel() * t.element_size() for t in inp.values() if isinstance(t, torch.Tensor))
    y = torch.empty(cfg.batch, cfg.seqlen, cfg.nheads, cfg.head_dim, dtype=torch.float32, device="meta")
    fs = torch.empty(cfg.batch, cfg.nheads, cfg.state_dim, cfg.head_dim, dtype=torch.float32, device="meta")
    return total + y.numel() * 4 + fs.numel() * 4


# the workloads at their own shapes where they are small, and shortened rows
# of the large ones (every term keeps its form: G > 1, an initial state, D
# drawn per head)
CASES = [
    SCAN_CONFIGS["c0_tiny_fp32"],
    SCAN_CONFIGS["c1_130m"],
    SCAN_CONFIGS["c2_2p7b"].with_(batch=2, seqlen=512),
    SCAN_CONFIGS["c3_long"].with_(seqlen=1024),
]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: "%s_b%d_L%d" % (c.name, c.batch, c.seqlen))
def test_scan_bytes_are_the_tensors_one_call_moves(cfg):
    assert bench.scan_bytes(cfg) == _scan_tensor_bytes(cfg)


def test_scan_bytes_scale_with_tokens():
    """Only the state and parameter terms are per call: doubling the tokens
    of a workload adds exactly one more token slab."""
    c = SCAN_CONFIGS["c3_long"]
    one = bench.scan_bytes(c.with_(seqlen=1024))
    two = bench.scan_bytes(c.with_(seqlen=2048))
    full = bench.scan_bytes(c)
    slab = two - one
    assert full == pytest.approx(one + slab * (c.seqlen // 1024 - 1), rel=0, abs=0)


def _chunked_flops_by_enumeration(b, L, H, P, N, G, Q):
    """2 flops per multiply-add, every chunk padded to Q tokens."""
    nc = math.ceil(L / Q)
    per_chunk_group = 0
    per_chunk_head = 0
    for i in range(Q):
        for j in range(Q):
            if j <= i:
                per_chunk_group += 2 * N          # (C.B^T)[i, j]
                per_chunk_head += 2 * P           # W[i, j] x_j into y_i
    per_chunk_head += 2 * Q * N * P               # chunk state B^T (w x)
    per_chunk_head += 2 * Q * N * P               # C_i . h for every token
    return b * nc * (G * per_chunk_group + H * per_chunk_head)


@pytest.mark.parametrize("shape", [(1, 32, 2, 2, 3, 1, 4), (2, 48, 4, 3, 5, 2, 8), (1, 64, 6, 4, 2, 3, 16)])
def test_scan_flops_count_the_causal_chunked_form(shape):
    b, L, H, P, N, G, Q = shape
    cfg = SCAN_CONFIGS["c1_130m"].with_(batch=b, seqlen=L, nheads=H, head_dim=P, state_dim=N, ngroups=G,
                                       chunk_size=Q)
    assert bench.scan_flops(cfg) == _chunked_flops_by_enumeration(b, L, H, P, N, G, Q)


def test_step_bytes_are_the_tensors_one_step_moves():
    """The decode step reads and writes the state once each, reads one token's
    x, B, C, dt_raw and the per-head parameters, writes y (fp32)."""
    cfg = STEP_CONFIGS["c4_decode"].with_(batch=4)
    inp = make_step_inputs(cfg, steps=1)
    state = inp["state"]
    total = 2 * state.numel() * state.element_size()
    total += sum(inp[k].numel() * inp[k].element_size() for k in ("x", "B", "C", "dt_raw", "dt_bias", "A", "D"))
    total += cfg.batch * cfg.nheads * cfg.head_dim * 4
    assert bench.step_bytes(cfg) == total
