"""GPU parity of packed rows (ssd_chunk_scan_fwd_varlen, SIMT path) against
the fp64 oracle: documents restart from a zero state at every start (a
token whose seq_idx differs from the previous one's).  Bars as for the
scan: 1e-4 (fp32 inputs) and 2e-2 (bf16 inputs) of RMS for y and
final_state; each chunk-boundary state against its own RMS."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import TOL_BF16, compare, path_supported, run_scan, to_dev, tol_for
from state_space_sequence_scan_b200 import ssd
from state_space_sequence_scan_b200.inputs import SCAN_CONFIGS, ScanConfig, make_scan_inputs
from test_gpu_states import compare_states

pytestmark = pytest.mark.gpu


def _seq_idx(b, L, rng, mean_len, Q):
    """Random document lengths (down to one token), one start put exactly on
    a chunk boundary in each row."""
    seq = np.zeros((b, L), np.int32)
    for bi in range(b):
        cuts = set(int(c) for c in rng.integers(1, L, size=max(1, L // mean_len)))
        if Q < L:
            cuts.add(Q)
        cuts.update({5, 6})                      # a one-token document
        doc = 0
        for t in range(L):
            if t in cuts:
                doc += 1
            seq[bi, t] = doc
    return seq


def _run(inp, seq, Q, states=False, path="auto"):
    d = to_dev(inp)
    y, fs, cs = ssd.chunk_scan_fwd_varlen(d["x"], d["dt_raw"], d["dt_bias"], d["A"], d["B"], d["C"], d["D"],
                                          torch.from_numpy(seq).cuda(), init_state=d["init_state"], chunk_size=Q,
                                          path=path, want_chunk_states=states)
    torch.cuda.synchronize()
    out = [y.cpu().double().numpy(), fs.cpu().double().numpy()]
    out.append(cs.cpu().double().numpy() if cs is not None else None)
    return out


CASES = [
    # b, L, H, P, N, G, Q, dtype
    (2, 300, 4, 64, 128, 2, 64, "f32"),
    (2, 300, 4, 64, 128, 2, 256, "bf16"),
    (3, 77, 2, 16, 16, 1, 7, "f32"),
    (1, 40, 2, 8, 4, 2, 1, "f32"),
]


CASES += [
    (2, 700, 4, 64, 128, 2, 128, "bf16"),                # tensor path: starts inside and on block edges
    (1, 549, 8, 64, 128, 1, 64, "bf16"),
]


@pytest.mark.parametrize("path", ["simt", "tensor"])
@pytest.mark.parametrize("states", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "b%d_L%d_H%d_P%d_N%d_G%d_Q%d_%s" % c)
def test_packed_parity(case, states, path):
    b, L, H, P, N, G, Q, dtype = case
    cfg = ScanConfig("packed", b, L, H, P, N, G, Q, dtype, "normal", "normal", seed=70 + L)
    inp = make_scan_inputs(cfg)
    if not path_supported(inp, Q, path) or (path == "tensor" and states and Q % 128):
        pytest.skip("the %s path does not take this shape" % path)
    seq = _seq_idx(b, L, np.random.default_rng(L + Q), 23, Q)
    y, fs, cs = _run(inp, seq, Q, states, path)
    yr, fr, sr = oracle.scan_varlen(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                                    seq, chunk_size=Q, init_state=inp["init_state"])
    tol = tol_for(inp["x"].dtype)
    compare(y, yr, tol, "packed y")
    compare(fs, fr, tol, "packed final_state")
    if states:
        compare_states(cs, sr, tol, "packed chunk states")
        assert np.array_equal(cs[:, -1], fs)


def test_one_document_is_the_plain_scan_bit_for_bit():
    """Constant ids: every mask passes, so the arithmetic is the plain SIMT
    scan's, to the bit."""
    cfg = ScanConfig("one", 2, 200, 4, 32, 32, 2, 64, "f32", "normal", "normal", seed=80)
    inp = make_scan_inputs(cfg)
    y, fs, _ = _run(inp, np.full((2, 200), 3, np.int32), 64)
    y0, fs0 = run_scan(inp, 64, path="simt")
    assert np.array_equal(y, y0) and np.array_equal(fs, fs0)


def test_one_document_tensor_path_is_the_plain_scan_bit_for_bit():
    cfg = ScanConfig("one_tc", 2, 700, 4, 64, 128, 2, 256, "bf16", "normal", "normal", seed=81)
    inp = make_scan_inputs(cfg)
    y, fs, _ = _run(inp, np.full((2, 700), 3, np.int32), 256, path="tensor")
    y0, fs0 = run_scan(inp, 256, path="tensor")
    assert np.array_equal(y, y0) and np.array_equal(fs, fs0)


@pytest.mark.parametrize("path", ["simt", "tensor"])
def test_packed_130m_shaped_rows(path):
    """The 130m-shaped layer packed into documents of about 300 tokens, every
    chain against the oracle."""
    cfg = SCAN_CONFIGS["c1_130m"]
    inp = make_scan_inputs(cfg)
    seq = _seq_idx(cfg.batch, cfg.seqlen, np.random.default_rng(5), 300, cfg.chunk_size)
    y, fs, _ = _run(inp, seq, cfg.chunk_size, path=path)
    yr, fr, _ = oracle.scan_varlen(inp["x"], inp["dt_raw"], inp["dt_bias"], inp["A"], inp["B"], inp["C"], inp["D"],
                                   seq, chunk_size=cfg.chunk_size, init_state=inp["init_state"])
    compare(y, yr, TOL_BF16, "packed 130m y")
    compare(fs, fr, TOL_BF16, "packed 130m final_state")


def test_packed_long_context_units():
    """The long-context layer (units of 47 blocks: the unit passes carry the
    resets) packed into documents of about 4000 tokens; every fifth head
    against the oracle, the bar over all of them."""
    from gpu_helpers import StreamingCompare, stack_chains
    cfg = SCAN_CONFIGS["c3_long"]
    inp = make_scan_inputs(cfg)
    seq = _seq_idx(cfg.batch, cfg.seqlen, np.random.default_rng(6), 4000, cfg.chunk_size)
    y, fs, _ = _run(inp, seq, cfg.chunk_size, path="tensor")
    chains = [(0, h) for h in range(0, cfg.nheads, 5)]
    sub = stack_chains(inp, chains)
    yr, fr, _ = oracle.scan_varlen(sub["x"], sub["dt_raw"], sub["dt_bias"], sub["A"], sub["B"], sub["C"], sub["D"],
                                   seq[:1], chunk_size=cfg.chunk_size, init_state=sub["init_state"])
    cy, cf = StreamingCompare(TOL_BF16, "packed c3 y"), StreamingCompare(TOL_BF16, "packed c3 final_state")
    for j, (bi, h) in enumerate(chains):
        cy.add(y[bi, :, h], yr[0, :, j])
        cf.add(fs[bi, h], fr[0, j])
    cy.check()
    cf.check()
