"""Helpers shared by the GPU parity tests: host <-> device conversion and the
acceptance checks (routing exact outside near-ties, gates to 1e-3, layer output
to rel-L2 1e-2 / max-abs 5e-2)."""
import numpy as np

import moe_inputs as mi

MARGIN = 1e-3       # tokens whose k-th / (k+1)-th biased-score gap is below this are exempt
GATE_ATOL = 1e-3
OUT_REL_L2 = 1e-2
OUT_MAX_ABS = 5e-2


def dev_bf16(u16):
    import torch

    return torch.from_numpy(np.ascontiguousarray(u16).view(np.int16)).view(torch.bfloat16).cuda()


def host_bf16_f64(t):
    import torch

    return mi.bf16_to_f64(t.detach().view(torch.int16).cpu().numpy().view(np.uint16))


def host_bf16_bits(t):
    import torch

    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def check_routing(gpu_idx, gpu_gates, gpu_counts, ref, k, n_routed, n_shared, gate_scale=1.0):
    """Compare the GPU router with the oracle; returns the mask of tokens whose
    GPU selection equals the oracle's (as a set).

    * tokens with oracle margin >= MARGIN: same set of experts, bit for bit;
      same order where every gap between consecutive kept scores is >= MARGIN
    * every token: gates within GATE_ATOL (times the gate scale) of the oracle's
      gates for the same expert ids (for exempt tokens whose set differs: the GPU
      gates sum to the scale)
    * counts: equal to the histogram of the GPU's own selection; equal to the
      oracle's where no token is exempt, else within the number of exempt tokens
    """
    exempt = ref["margin"] < MARGIN
    same = (np.sort(gpu_idx, axis=1) == np.sort(ref["topk_idx"], axis=1)).all(axis=1)
    bad = ~same & ~exempt
    assert not bad.any(), f"{bad.sum()} non-exempt tokens select different experts, e.g. token {np.argmax(bad)}"
    # order, where the oracle's kept scores are well separated
    sel_sorted = np.take_along_axis(ref["sel"], ref["topk_idx"].astype(np.int64), axis=1)
    gaps_ok = (np.diff(-sel_sorted, axis=1) >= MARGIN).all(axis=1) & ~exempt
    assert (gpu_idx[gaps_ok] == ref["topk_idx"][gaps_ok]).all()
    # gates per expert id: both sides' (id, gate) pairs sorted by id (the sets are equal on these tokens)
    ts = np.nonzero(same)[0]
    ids = np.concatenate([gpu_idx[ts], np.broadcast_to(np.arange(n_routed, n_routed + n_shared),
                                                       (len(ts), n_shared))], axis=1)
    o_gpu = np.argsort(ids, axis=1, kind="stable")
    o_ref = np.argsort(ref["contrib"][ts], axis=1, kind="stable")
    np.testing.assert_array_equal(np.take_along_axis(ids, o_gpu, 1), np.take_along_axis(ref["contrib"][ts], o_ref, 1))
    g_gpu = np.take_along_axis(gpu_gates[ts], o_gpu, 1)
    g_ref = np.take_along_axis(ref["gates"][ts], o_ref, 1)
    err = np.abs(g_gpu - g_ref)
    assert (err <= GATE_ATOL * gate_scale).all(), f"gate error {err.max():.3e} at token {ts[np.argmax(err.max(1))]}"
    np.testing.assert_allclose(gpu_gates.sum(axis=1), gate_scale, atol=1e-5 * gate_scale)
    # counts
    own = np.bincount(gpu_idx.reshape(-1), minlength=n_routed)
    np.testing.assert_array_equal(gpu_counts, own)
    ref_counts = np.bincount(ref["topk_idx"].reshape(-1), minlength=n_routed)
    n_ex = int(exempt.sum())
    if not (~same).any():
        np.testing.assert_array_equal(gpu_counts, ref_counts)
    else:
        assert np.abs(gpu_counts.astype(np.int64) - ref_counts).max() <= n_ex
    return same


def check_output(gpu_out, ref_out, label=""):
    diff = gpu_out - ref_out
    rel = np.linalg.norm(diff) / max(np.linalg.norm(ref_out), 1e-30)
    mx = np.abs(diff).max() if diff.size else 0.0
    assert rel <= OUT_REL_L2, f"{label}: rel-L2 {rel:.3e}"
    assert mx <= OUT_MAX_ABS, f"{label}: max-abs {mx:.3e}"
    return rel, mx
