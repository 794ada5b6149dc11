"""Shared helpers of the GPU parity tests: run a workload through the C ABI and
compare it with the CPU oracle decision by decision.

Decision parity (the contract of the tests): for every sequence, the accepted
count and every emitted token must equal the oracle's, except where the
oracle's margin at the first differing decision is below ``MARGIN``:
|u_accept - ratio| for an acceptance test, and for the draw the distance of
u_resample to the ends of the chosen token's interval of the normalised
cumulative mass.  Such cases are counted and reported.  Softmax quantities
must agree within ``PROB_TOL`` absolute (q(t), p(t), residual mass Z) and the
log normalisers log sum_i exp(x_i/T) within ``LSE_TOL`` absolute.
"""
from __future__ import annotations

import os

import numpy as np

MARGIN = 1e-6
PROB_TOL = 1e-5
LSE_TOL = 1e-5   # absolute, i.e. relative on the normaliser
# A residual draw is determined at the kernels' precision only when the
# residual mass Z is well above the rounding of q - p: the fp32 normalisers
# agree with the oracle's to about 1e-7, so below Z = 1e-6 the residual's
# relative error passes 10% (the oracle's own Z there is often fp64 rounding,
# e.g. 1e-80 when q and p are nearly the same point mass).  Such draws are
# checked for validity only and reported as "unresolved".
RESID_RESOLVE = 1e-6


def _unresolved(ora, b, no, G):
    return no < G and float(ora["resid_mass"][b]) < RESID_RESOLVE


def _valid_draw(tg, no, V, logit_row=None, top_k=0):
    """The emitted token lies in [0, V), everything after it is -1 and (given the
    target row) its logit is finite and not below the k-th largest."""
    tok = int(tg[no])
    if not (0 <= tok < V) or not (np.asarray(tg[no + 1:]) == -1).all():
        return False
    if logit_row is None:
        return True
    x = np.asarray(logit_row, np.float32)
    if not np.isfinite(x[tok]):
        return False
    return not (0 < top_k < V) or x[tok] >= np.partition(x, V - top_k)[V - top_k]


# A residual entry max(0, q - p) is formed in fp32 on the GPU: where q and p
# agree to about this relative precision its sign is not determined.
RESID_SIGN_TOL = 1e-6


def _residual_token_ok(target_row, draft_row, T, tok, fallback):
    """An unresolved residual draw must still come from the residual's support
    at the kernels' precision: q_n(tok) > 0 and q_n(tok) - p_n(tok) not below
    -RESID_SIGN_TOL of the larger of the two (oracle softmaxes of the rejected
    position's rows).  Under the zero-mass fallback the draw is from q_n, so
    q_n(tok) > 0 is enough.  A token from the wrong row, or one the draft
    favours clearly (q < p), fails."""
    import oracle
    q = oracle.softmax(np.ascontiguousarray(target_row), T)[0][tok]
    if not q > 0.0:
        return False
    if fallback:
        return True
    p = oracle.softmax(np.ascontiguousarray(draft_row), T)[0][tok]
    return q - p >= -RESID_SIGN_TOL * max(q, p)


# parity counts of every comparison in this process, printed at the end of the
# test session (tests/conftest.py) so that a quiet run still reports them
REPORT: list = []


def record(summary, name=None):
    """Keep the counts of one comparison for the end-of-session report."""
    REPORT.append((name or summary.get("name", "?"), summary["sequences"], len(summary["hard"]),
                   len(summary["margin_cases"]), len(summary["unresolved"])))
    return summary


def to_device(wl, device=0):
    import torch
    dev = torch.device("cuda", device)

    def logits(a):
        if wl.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    out = {}
    if getattr(wl, "mapped", False):
        m = wl.meta
        out = {"target_rows": logits(m["target_rows"]),
               "target_map": torch.from_numpy(np.ascontiguousarray(m["target_map"], np.int32)).to(dev),
               "draft_rows": logits(m["draft_rows"]),
               "draft_map": torch.from_numpy(np.ascontiguousarray(m["draft_map"], np.int32)).to(dev)}
    return out | {
        "target": logits(wl.target),
        "draft": logits(wl.draft),
        "tokens": torch.from_numpy(np.ascontiguousarray(wl.tokens, np.int32)).to(dev),
        "u_accept": torch.from_numpy(np.ascontiguousarray(wl.u_accept, np.float32)).to(dev),
        "u_resample": torch.from_numpy(np.ascontiguousarray(wl.u_resample, np.float32)).to(dev),
    }


def gpu_run(wl, slices=None, threads=None, device=0, inputs=None, sv=None, readback=True,
            mapped=False, fused=None):
    """One verification call of the whole workload; returns numpy outputs.

    ``mapped``: call the shared-row entry point on the workload's distinct rows
    and row maps instead of the per-position arrays.  ``fused``: True or a
    (unit_groups, chunk_tiles, lag) tuple selects the single-launch form,
    False the three kernels; None keeps the handle's setting."""
    import torch
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    own = sv is None
    if own:
        sv = SpecVerify(wl.batch, wl.gamma, wl.vocab, wl.dtype, device)
    try:
        if slices is not None or threads is not None:
            c0, t0 = sv.launch()
            sv.set_launch(min(slices or c0, sv.max_slices), threads or t0)
        if fused is not None:
            if isinstance(fused, tuple):
                sv.set_fused(True, *fused)
            else:
                sv.set_fused(bool(fused))
        d = inputs if inputs is not None else to_device(wl, device)
        out_t = torch.full((wl.batch, wl.gamma + 1), -7, dtype=torch.int32, device=f"cuda:{device}")
        out_n = torch.full((wl.batch,), -7, dtype=torch.int32, device=f"cuda:{device}")
        if mapped:
            sv.run_mapped(d["target_rows"], d["target_map"], d["draft_rows"], d["draft_map"],
                          d["tokens"], d["u_accept"], d["u_resample"], wl.temperature, out_t,
                          out_n)
        else:
            sv.run(d["target"], d["draft"], d["tokens"], d["u_accept"], d["u_resample"],
                   wl.temperature, out_t, out_n)
        torch.cuda.synchronize(device)
        status, bits = sv.status()
        res = {"out_tokens": out_t.cpu().numpy(), "out_num_accepted": out_n.cpu().numpy(),
               "status": status, "bits": bits, "launch": sv.launch()}
        if readback:
            res.update(sv.readback())
        return res
    finally:
        if own:
            sv.close()


def oracle_run(wl, b_range=None):
    import oracle
    # the C ABI takes the temperature as a float: the oracle gets the same value
    return oracle.verify(wl.target, wl.draft, wl.tokens, wl.u_accept, wl.u_resample,
                         float(np.float32(wl.temperature)), threads=os.cpu_count() or 1,
                         b_range=b_range)


def compare(wl, gpu, ora, seqs=None, check_probs=True, logits=None):
    """Decision parity over the sequences `seqs` (default: all).  Returns a summary dict.

    ``logits``: the (target, draft) logit arrays the oracle ran on, when they
    are not ``wl.target`` / ``wl.draft`` (the LM-head-fused step's float64
    logits); an unresolved residual draw is checked against their softmaxes."""
    B, G = wl.batch, wl.gamma
    seqs = np.arange(B) if seqs is None else np.asarray(seqs)
    tgt_all, drf_all = logits if logits is not None else (wl.target, wl.draft)
    T = float(np.float32(wl.temperature))
    hard, margin_cases, unresolved = [], [], []
    for b in seqs:
        ng, no = int(gpu["out_num_accepted"][b]), int(ora["out_num_accepted"][b])
        tg, to = gpu["out_tokens"][b], ora["out_tokens"][b]
        if ora["seq_status"][b] in (16, 17):
            if ng != 0 or not (tg == -1).all():
                hard.append((int(b), "error outcome", ng, tg.tolist()))
            continue
        if ng != no:
            j = min(ng, no)
            m = ora["accept_margin"][b, j]
            (margin_cases if m < MARGIN else hard).append((int(b), "accept", j, float(m)))
            continue
        if not np.array_equal(tg, to):
            # the zero-mass fallback draws from q_n, which is resolved: it is
            # compared like any other draw
            if _unresolved(ora, b, no, G) and ora["seq_status"][b] != 18:
                ok_draw = (np.array_equal(tg[:no], to[:no]) and _valid_draw(tg, no, wl.vocab)
                           and _residual_token_ok(tgt_all[b, no], drf_all[b, no], T, int(tg[no]),
                                                  False))
                (unresolved if ok_draw else hard).append(
                    (int(b), "unresolved draw", int(tg[no]), int(to[no]), float(ora["resid_mass"][b])))
                continue
            m = ora["cdf_margin_norm"][b]
            (margin_cases if m < MARGIN else hard).append(
                (int(b), "draw", int(tg[no]), int(to[no]), float(m)))
    summary = {"name": wl.name, "sequences": int(len(seqs)), "hard": hard,
               "margin_cases": margin_cases, "unresolved": unresolved}
    if check_probs and "q_tok" in gpu:
        ok = ora["seq_status"][seqs] == 0
        s = seqs[ok]
        if G > 0 and len(s):
            tested = ~np.isnan(ora["q_tok"][s])
            dq = np.abs(gpu["q_tok"][s] - ora["q_tok"][s])[tested]
            dp = np.abs(gpu["p_tok"][s] - ora["p_tok"][s])[tested]
            summary["max_dq"] = float(dq.max()) if dq.size else 0.0
            summary["max_dp"] = float(dp.max()) if dp.size else 0.0
            # log sum_i exp(x_i/T) = max/T + log(sum) in the oracle's terms
            lse_d = ora["draft_max"][s] / wl.temperature + np.log(ora["draft_sum"][s])
            summary["max_draft_lse_abs"] = float(np.abs(gpu["draft_lse"][s] - lse_d).max())
        if len(s):
            lse_t = ora["target_max"][s] / wl.temperature + np.log(ora["target_sum"][s])
            summary["max_target_lse_abs"] = float(np.abs(gpu["target_lse"][s] - lse_t).max())
            dz = np.abs(gpu["resid_mass"][s] - ora["resid_mass"][s])
            summary["max_dz"] = float(np.nanmax(dz)) if dz.size else 0.0
    return summary


def assert_parity(summary, max_margin_frac=0.01, max_unresolved_frac=0.01, report=True):
    """Hard differences fail; margin cases and unresolved draws are each capped
    at a fraction of the sequences (at least one).  The counts are recorded
    for the end-of-session report first, so a failing comparison is reported
    too."""
    if report:
        record(summary)
    assert not summary["hard"], f"decisions differ outside the margin: {summary['hard'][:5]}"
    assert len(summary["margin_cases"]) <= max(1, max_margin_frac * summary["sequences"]), summary
    assert len(summary["unresolved"]) <= max(1, max_unresolved_frac * summary["sequences"]), summary
    for key in ("max_dq", "max_dp", "max_dz"):
        if key in summary:
            assert summary[key] <= PROB_TOL, summary
    for key in ("max_target_lse_abs", "max_draft_lse_abs"):
        if key in summary:
            assert summary[key] <= LSE_TOL, summary


FILTER_MARGIN = 1e-6   # top-p boundary: |cumulative mass - top_p| below this is a margin case


def gpu_run_sampling(wl, temperatures, top_k=0, top_p=1.0, device=0, inputs=None, sv=None):
    """One call of the sampling-variant entry point; numpy outputs plus readbacks."""
    import torch
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    own = sv is None
    if own:
        sv = SpecVerify(wl.batch, wl.gamma, wl.vocab, wl.dtype, device)
    try:
        d = inputs if inputs is not None else to_device(wl, device)
        temps = torch.from_numpy(np.array(
            np.broadcast_to(np.asarray(temperatures, np.float32), (wl.batch,)))).to(f"cuda:{device}")
        out_t = torch.full((wl.batch, wl.gamma + 1), -7, dtype=torch.int32, device=f"cuda:{device}")
        out_n = torch.full((wl.batch,), -7, dtype=torch.int32, device=f"cuda:{device}")
        sv.run_sampling(d["target"], d["draft"], d["tokens"], d["u_accept"], d["u_resample"],
                        temps, out_t, out_n, top_k=top_k, top_p=top_p)
        torch.cuda.synchronize(device)
        status, bits = sv.status()
        res = {"out_tokens": out_t.cpu().numpy(), "out_num_accepted": out_n.cpu().numpy(),
               "status": status, "bits": bits}
        res.update(sv.readback())
        res["kept_target"], res["kept_draft"] = sv.kept()
        return res
    finally:
        if own:
            sv.close()


def oracle_run_sampling(wl, temperatures, top_k=0, top_p=1.0):
    import oracle
    return oracle.verify_sampling(wl.target, wl.draft, wl.tokens, wl.u_accept, wl.u_resample,
                                  np.asarray(temperatures, np.float32), top_k=top_k,
                                  top_p=float(np.float32(top_p)), threads=os.cpu_count() or 1)


def _target_row(wl, b, n):
    from speculative_decoding_verification_90_b200 import workloads
    row = wl.target[b, n]
    return workloads.bits_to_f32(row) if wl.dtype == "bf16" else row


def compare_sampling(wl, gpu, ora, top_k=0):
    """Decision parity of the sampling variants.  A sequence with a row whose
    top-p boundary margin (|cumulative mass - top_p| at the chosen cut, relative
    to the kept mass) is below FILTER_MARGIN may cut one group differently: its
    kept counts and probabilities are not compared, and a differing decision
    counts as a margin case.  Everything else must agree as in the plain step."""
    B, G = wl.batch, wl.gamma
    hard, margin_cases, unresolved = [], [], []
    ok = []
    for b in range(B):
        ng, no = int(gpu["out_num_accepted"][b]), int(ora["out_num_accepted"][b])
        tg, to = gpu["out_tokens"][b], ora["out_tokens"][b]
        if ora["seq_status"][b] in (16, 17, 21):
            if ng != 0 or not (tg == -1).all():
                hard.append((b, "error outcome", ng, tg.tolist()))
            continue
        near_cut = ora["filter_margin"][b] < FILTER_MARGIN
        if not near_cut:
            if ora["seq_status"][b] == 0:
                ok.append(b)   # a zero-mass fallback's residual mass is rounding
            if not (np.array_equal(gpu["kept_target"][b], ora["kept_target"][b])
                    and np.array_equal(gpu["kept_draft"][b], ora["kept_draft"][b])):
                hard.append((b, "kept", gpu["kept_target"][b].tolist(),
                             ora["kept_target"][b].tolist()))
                continue
        if ng != no:
            j = min(ng, no)
            m = ora["accept_margin"][b, j]
            (margin_cases if (m < MARGIN or near_cut) else hard).append((b, "accept", j, float(m)))
            continue
        if not np.array_equal(tg, to):
            if _unresolved(ora, b, no, G):
                row = _target_row(wl, b, no)
                ok_draw = np.array_equal(tg[:no], to[:no]) and _valid_draw(tg, no, wl.vocab, row, top_k)
                (unresolved if ok_draw else hard).append(
                    (b, "unresolved draw", int(tg[no]), int(to[no]), float(ora["resid_mass"][b])))
                continue
            m = ora["cdf_margin_norm"][b]
            (margin_cases if (m < MARGIN or near_cut) else hard).append(
                (b, "draw", int(tg[no]), int(to[no]), float(m)))
    summary = {"name": wl.name + " (sampling)", "sequences": B, "hard": hard,
               "margin_cases": margin_cases, "unresolved": unresolved,
               "near_cut": int((ora["filter_margin"] < FILTER_MARGIN).sum())}
    s = np.asarray(ok, dtype=np.int64)
    if G > 0 and len(s):
        tested = ~np.isnan(ora["q_tok"][s])
        summary["max_dq"] = float(np.abs(gpu["q_tok"][s] - ora["q_tok"][s])[tested].max(initial=0.0))
        summary["max_dp"] = float(np.abs(gpu["p_tok"][s] - ora["p_tok"][s])[tested].max(initial=0.0))
    if len(s):
        dz = np.abs(gpu["resid_mass"][s] - ora["resid_mass"][s])
        summary["max_dz"] = float(np.nanmax(dz)) if dz.size else 0.0
    return summary
