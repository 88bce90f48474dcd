"""GPU parity: the CUDA kernels (through the C ABI) against the fp64 CPU oracle.

Tolerances (fixed for this operator): output max-abs <= 3e-2 and relative L2 <= 1e-2;
final state relative L2 <= 1e-2; every element finite.
"""
import numpy as np
import pytest
import torch

import kda_inputs
import kimi_delta_attention_24_b200 as kda
import margins
import oracle

pytestmark = pytest.mark.gpu

O_MAX_ABS = 3e-2
O_REL_L2 = 1e-2
S_REL_L2 = 1e-2
IMPLS = ["chunked", "recurrent"]


def rel_l2(a, b):
    nb = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (nb if nb > 0 else 1.0)


def run_gpu(x, impl="chunked", state_transposed=False, alias=False, dev="cuda:0"):
    xd = x.to(dev)
    B, T, H, K = xd.q.shape
    N = xd.num_seqs
    out = torch.full_like(xd.v, float("nan"))
    s0 = xd.initial_state
    if s0 is not None and state_transposed:
        s0 = s0.transpose(-1, -2).contiguous()
    final = None
    if x.output_final_state:
        final = s0 if alias else torch.full((N, H, K, K), float("nan"), dtype=torch.float32, device=dev)
    ws = kda.new_workspace(B * T, H, N, dev)
    fn = kda.fwd if impl == "chunked" else kda.fwd_recurrent
    fn(xd.q, xd.k, xd.v, xd.g, xd.beta, xd.scale, out, ws, xd.A_log, xd.dt_bias, xd.lower_bound,
       s0, final, xd.cu_seqlens, state_transposed=state_transposed)
    assert kda.read_device_status(ws) == 0
    o = out.float().cpu().double().numpy()
    s = None if final is None else final.cpu().double().numpy()
    return o, s


def check(o, s, o_ref, s_ref, what=""):
    """Asserts the parity tolerances and records the margins (printed at the end of the session)."""
    assert np.isfinite(o).all(), f"{what}: non-finite output"
    err = np.max(np.abs(o - o_ref)) if o.size else 0.0
    rl = rel_l2(o, o_ref)
    rs = None
    if s_ref is not None:
        assert np.isfinite(s).all(), f"{what}: non-finite state"
        rs = rel_l2(s, s_ref)
    margins.record(what, err, rl, rs)
    print(f"{what}: o max-abs {err:.3e}, o rel-L2 {rl:.3e}, state rel-L2 {rs if rs is None else f'{rs:.3e}'}")
    assert err <= O_MAX_ABS and rl <= O_REL_L2, f"{what}: o max-abs {err:.3e}, rel-L2 {rl:.3e}"
    if rs is not None:
        assert rs <= S_REL_L2, f"{what}: state rel-L2 {rs:.3e}"
    return err, rl


@pytest.mark.parametrize("impl", IMPLS)
@pytest.mark.parametrize("name", ["tiny", "tail", "varlen", "collinear", "usage"])
def test_workload_parity(cuda_device, name, impl):
    x = kda_inputs.make_workload(name)
    o_ref, s_ref = oracle.fwd_inputs(x)
    o, s = run_gpu(x, impl)
    check(o, s, o_ref, s_ref, f"{name}/{impl}")


@pytest.mark.parametrize("impl", IMPLS)
def test_prefill_sampled_heads(cuda_device, impl):
    """The 32K x 96-head prefill, in the bench's launch configuration; the oracle recomputes a
    sample of heads over the whole sequence."""
    x = kda_inputs.make_workload("prefill", device=cuda_device)
    if impl == "chunked":
        assert kda.fwd_launch_count(x.total_tokens, x.num_heads, x.num_seqs) == 5  # two stages
    o, s = run_gpu(x, impl)
    heads = [0, 41, 95]
    sl = lambda t: t[:, :, heads].contiguous().cpu()
    o_ref, s_ref = oracle.kda_fwd(sl(x.q), sl(x.k), sl(x.v), sl(x.g), sl(x.beta), x.scale,
                                  x.A_log[heads].cpu(), x.dt_bias[heads].cpu(), x.lower_bound,
                                  initial_state=x.initial_state[:, heads].cpu(),
                                  cu_seqlens=x.cu_seqlens.cpu())
    check(o[:, :, heads], s[:, heads], o_ref, s_ref, f"prefill/{impl}")


@pytest.mark.parametrize("T,H", [(8192, 64), (4096, 160)])
def test_other_head_counts_sampled(cuda_device, T, H):
    """One long sequence at 64 heads (two stages, another cut) and at 160 heads (more units than
    SMs: one stage); the oracle recomputes three heads over the whole sequence."""
    x = kda_inputs.make_random("t", [T], H, seed=35, state_std=0.1, device=cuda_device)
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    assert kda.fwd_launch_count(T, H, 1) == (5 if H < sms else 3)
    o, s = run_gpu(x, "chunked")
    heads = [0, H // 2, H - 1]
    sl = lambda t: t[:, :, heads].contiguous().cpu()
    o_ref, s_ref = oracle.kda_fwd(sl(x.q), sl(x.k), sl(x.v), sl(x.g), sl(x.beta), x.scale,
                                  x.A_log[heads].cpu(), x.dt_bias[heads].cpu(), x.lower_bound,
                                  initial_state=x.initial_state[:, heads].cpu(),
                                  cu_seqlens=x.cu_seqlens.cpu())
    check(o[:, :, heads], s[:, heads], o_ref, s_ref, f"T={T} H={H}")


def test_chunk_tails_and_empty_documents(cuda_device):
    lens = [1, 2, 15, 16, 17, 0, 63, 64, 65, 0, 127, 128, 129, 200]
    x = kda_inputs.make_random("t", lens, 2, seed=21, state_std=0.2)
    o_ref, s_ref = oracle.fwd_inputs(x)
    for impl in IMPLS:
        o, s = run_gpu(x, impl)
        check(o, s, o_ref, s_ref, f"tails/{impl}")
    # zero-length documents hand their initial state through
    np.testing.assert_array_equal(s[5], x.initial_state[5].double().numpy())


@pytest.mark.parametrize("opt", ["plain", "transposed", "no_final", "alias"])
def test_two_stage_schedule(cuda_device, opt):
    """N * H below the SM count: the chunk range runs in two stages (five launches) and the
    document holding the cut hands its state from the first recurrence launch to the second
    through the workspace; empty documents sit on both sides of the cut."""
    lens = [1000, 0, 2048, 77, 1, 3000, 0]
    assert kda.fwd_launch_count(sum(lens), 4, len(lens)) == 5
    x = kda_inputs.make_random("t", lens, 4, seed=32, state_std=0.1,
                               output_final_state=opt != "no_final")
    o_ref, s_ref = oracle.fwd_inputs(x, state_transposed=opt == "transposed")
    o, s = run_gpu(x, "chunked", state_transposed=opt == "transposed", alias=opt == "alias")
    check(o, s, o_ref, s_ref, f"two stages/{opt}")


def _stage_cut(lens, H, sms):
    """Where the launcher cuts the global chunk range (its documented sizing rule), or None."""
    T, N = sum(lens), len(lens)
    mc = (T + 63 * N) // 64
    if N * H >= sms:
        return None
    x = 0.45 * (sms - N * H) / H
    g = mc - int(mc * x / (1 + x))
    return g if 0 < g < mc else None


def _cut_layouts(H, sms):
    """Seeded document layouts whose stage cut falls exactly on a document start, inside a
    document, and on an empty document."""
    rng = np.random.default_rng(33)
    found = {}
    for _ in range(20000):
        n = int(rng.integers(2, 7))
        lens = [int(v) * 64 + (int(rng.integers(0, 64)) if rng.random() < 0.3 else 0)
                for v in rng.integers(0, 9, size=n)]
        if sum(lens) == 0:
            continue
        g = _stage_cut(lens, H, sms)
        if g is None:
            continue
        co = np.concatenate([[0], np.cumsum([(L + 63) // 64 for L in lens])])
        if any(co[i] == g == co[i + 1] for i in range(n)):
            kind = "empty document at the cut"
        elif any(co[i] < g < co[i + 1] for i in range(n)):
            kind = "cut inside a document"
        elif g in co:
            kind = "cut on a document start"
        else:
            continue
        found.setdefault(kind, lens)
        if len(found) == 3:
            break
    return found


def test_stage_cut_positions(cuda_device):
    """The two-stage schedule with the cut on a document start (no hand-over), inside a
    document (state handed over through the workspace) and on an empty document."""
    H = 2
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    layouts = _cut_layouts(H, sms)
    assert len(layouts) == 3, layouts
    for kind, lens in layouts.items():
        assert kda.fwd_launch_count(sum(lens), H, len(lens)) == 5
        x = kda_inputs.make_random("t", lens, H, seed=34, state_std=0.1)
        o_ref, s_ref = oracle.fwd_inputs(x)
        check(*run_gpu(x), o_ref, s_ref, f"{kind} {lens}")


# Byte layout of one (chunk, head) item that the intra-chunk kernel leaves in the workspace (an
# internal format: the test decodes it to check each stage against the fp64 chunked form).
_WS_HEADER, _ITEM = 256, 82944
_IT_WQ, _IT_TP, _IT_TL, _IT_KT, _IT_IK, _IT_GAM = 0, 32768, 49152, 65536, 81920, 82176


def _bf16_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _swizzled_tile(raw, rows):
    """[rows][64] bf16 from a 128-byte-swizzled image: row r's 16-byte chunk c is stored at c ^ (r % 8)."""
    u = np.frombuffer(raw, dtype=np.uint16).reshape(rows, 8, 8)
    r = np.arange(rows)[:, None]
    c = np.arange(8)[None, :]
    return _bf16_to_f64(u[r, c ^ (r & 7)].reshape(rows, 64))


def _stage_case(case):
    """Inputs of the stage-level checks: random documents with a 2-token tail, the first four
    chunks of the near-collinear stress case, and saturated gates (log alpha = lower_bound on every
    channel) with beta = 1."""
    if case == "random":
        return kda_inputs.make_random("t", [130, 64], 2, seed=41, state_std=0.1)
    if case == "collinear":
        x = kda_inputs.make_workload("collinear")
        T = 256
        sl = lambda t: t[:, :T].contiguous()
        return kda_inputs.KDAInputs("collinear256", sl(x.q), sl(x.k), sl(x.v), sl(x.g), sl(x.beta),
                                    x.A_log, x.dt_bias, x.lower_bound, x.scale, x.initial_state,
                                    torch.tensor([0, T], dtype=torch.int32))
    if case == "saturated":
        x = kda_inputs.make_random("t", [192, 70], 2, seed=42, state_std=0.1)
        x.g.fill_(60.0)
        x.beta.fill_(30.0)
        return x
    raise KeyError(case)


# Stage tolerances (relative L2 against the fp64 chunked form; Qtil - P W against ||Qtil||).
# Random inputs: bf16 operands and outputs (-W, Qtil - P W, P T_b with P in bf16: a few 1e-3),
# hi + lo pairs on the fp32 / 3xTF32 solve (T_b: ~6e-5), fp32 scalars (1/|k|: ~4e-8, e^Gamma_C:
# ~5e-6).  Near-collinear keys: the rows of W beyond the first cancel to a small fraction of the
# first, so -W keeps bf16's absolute error on a smaller norm, and Qtil - P W cancels almost to
# zero (hence the norm of its terms); T_b is an fp32-accurate solve whatever the conditioning.
STAGE_TOL = {
    "random": {"-W": 1e-2, "Qtil - P W": 1e-2, "T_b": 1e-3, "P T_b": 2e-2, "Ktil": 5e-3,
               "1/|k|": 1e-6, "e^Gamma_C": 1e-4},
    "collinear": {"-W": 2e-2, "Qtil - P W": 2e-2, "T_b": 1e-3, "P T_b": 2e-2, "Ktil": 5e-3,
                  "1/|k|": 1e-6, "e^Gamma_C": 1e-4},
    "saturated": {"-W": 1e-2, "Qtil - P W": 1e-2, "T_b": 1e-3, "P T_b": 2e-2, "Ktil": 5e-3,
                  "1/|k|": 1e-6, "e^Gamma_C": 1e-4},
}


@pytest.mark.parametrize("case", ["random", "collinear", "saturated"])
def test_intra_chunk_stages_against_chunked_form(cuda_device, case):
    """Each intra-chunk output against the fp64 chunked form of the same chunk: -W and Qtil - P W
    (the MMA1 operand), T diag(beta) and P T diag(beta) (hi + lo pairs), Ktil (raw k with the decay
    to the chunk end), 1/|k| and e^{Gamma_C}; full chunks and partial tails."""
    from oracle.chunked import chunk_intermediates
    x = _stage_case(case)
    H = x.num_heads
    N = x.num_seqs
    xd = x.to(cuda_device)
    ws = kda.new_workspace(x.total_tokens, H, N, cuda_device)
    out = torch.empty_like(xd.v)
    kda.fwd(xd.q, xd.k, xd.v, xd.g, xd.beta, x.scale, out, ws, xd.A_log, xd.dt_bias, x.lower_bound,
            None, None, xd.cu_seqlens)
    assert kda.read_device_status(ws) == 0
    raw = ws.cpu().numpy().tobytes()
    cu = x.cu_seqlens.numpy()
    co = np.frombuffer(raw[_WS_HEADER:_WS_HEADER + 4 * (N + 1)], dtype=np.int32)
    assert list(co) == list(np.concatenate([[0], np.cumsum([(int(cu[i + 1] - cu[i]) + 63) // 64
                                                             for i in range(N)])]))
    items = _WS_HEADER + ((N + 1) * 4 + 1023) // 1024 * 1024
    qh, kh, la, be = oracle.prologue(x.q, x.k, x.g, x.beta, x.A_log, x.dt_bias, x.lower_bound)
    kraw = x.k.double().numpy()
    worst = {}
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            chunks = chunk_intermediates(qh[0, t0:t1, h], kh[0, t0:t1, h], x.v[0, t0:t1, h].double().numpy(),
                                         la[0, t0:t1, h], be[0, t0:t1, h], x.scale, 64)
            for c, ref in enumerate(chunks):
                L = ref["T"].shape[0]
                off = items + ((int(co[n]) + c) * H + h) * _ITEM
                it = raw[off:off + _ITEM]
                wq = np.concatenate([_swizzled_tile(it[_IT_WQ + 16384 * kb:_IT_WQ + 16384 * (kb + 1)], 128)
                                     for kb in range(2)], axis=1)
                tb = _swizzled_tile(it[_IT_TP:_IT_TP + 16384], 128) + _swizzled_tile(it[_IT_TL:_IT_TL + 16384], 128)
                kt = np.concatenate([_swizzled_tile(it[_IT_KT + 8192 * kb:_IT_KT + 8192 * (kb + 1)], 64)
                                     for kb in range(2)], axis=1)
                ik = np.frombuffer(it[_IT_IK:_IT_IK + 256], dtype=np.float32).astype(np.float64)
                gam = np.frombuffer(it[_IT_GAM:_IT_GAM + 512], dtype=np.float32).astype(np.float64)
                b = be[0, t0 + 64 * c:t0 + 64 * c + L, h]
                Tb = ref["T"] * b[None, :]
                kr = kraw[0, t0 + 64 * c:t0 + 64 * c + L, h]
                ik_ref = 1.0 / np.sqrt((kr * kr).sum(axis=1) + 1e-6)
                # (got, want, norm the error is measured against): Qtil - P W is a difference whose
                # terms cancel on nearly collinear keys (P W predicts Qtil almost exactly), so its
                # error is measured against the size of its terms, ||Qtil||; the others against
                # their own size
                qpw = ref["Qt"] - ref["P"] @ ref["W"]
                pairs = {
                    "-W": (wq[:L], -ref["W"], None),
                    "Qtil - P W": (wq[64:64 + L], qpw, max(np.linalg.norm(qpw), np.linalg.norm(ref["Qt"]))),
                    "T_b": (tb[:L, :L], Tb, None),
                    "P T_b": (tb[64:64 + L, :L], ref["P"] @ Tb, None),
                    "Ktil": (kt[:L], ref["Kt"] / ik_ref[:, None], None),
                    "1/|k|": (ik[:L], ik_ref, None),
                    # e^{Gamma_C} is a float32 product of decays: where the exact value is below
                    # float32's normal range (64 saturated decays: e^-320) it is zero
                    "e^Gamma_C": (gam, np.where(ref["gC"] < np.finfo(np.float32).tiny, 0.0, ref["gC"]), None),
                }
                assert np.all(ik[L:] == 0)  # rows past the end of the document
                for name, (got, want, nrm) in pairs.items():
                    assert np.isfinite(got).all(), name
                    err = rel_l2(got, want) if nrm is None else np.linalg.norm(got - want) / max(nrm, 1e-300)
                    worst[name] = max(worst.get(name, 0.0), err)
    print(f"stages/{case}: " + ", ".join(f"{k} {v:.2e}" for k, v in worst.items()))
    for name, err in worst.items():
        margins.note(f"stage {case} {name}: rel-L2 {err:.2e} (tol {STAGE_TOL[case][name]:.0e})")
    for name, err in worst.items():
        assert err <= STAGE_TOL[case][name], f"{case} {name}: rel-L2 {err:.3e}"


def test_launch_count_follows_the_stage_rule(cuda_device):
    """Two stages (5 launches) while N * H is below the SM count, one stage (3) from there on,
    2 when there are no tokens (chunk table and recurrence only), 0 without units."""
    sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    assert kda.fwd_launch_count(32768, 96, 1) == 5
    assert kda.fwd_launch_count(32768, sms, 1) == 3
    assert kda.fwd_launch_count(4096, 32, 8) == (3 if 32 * 8 >= sms else 5)
    assert kda.fwd_launch_count(0, 4, 1) == 2
    assert kda.fwd_launch_count(100, 0, 1) == 0
    assert kda.fwd_launch_count(100, 4, 0) == 0
    assert kda.fwd_launch_count(64, 1, 1) == 3  # a single chunk: nothing to cut


def test_many_short_documents(cuda_device):
    """1100 documents of 0..70 tokens: the per-sequence chunk table spans two 1024-wide scan
    blocks, and many chunks end a document part-way."""
    rng = np.random.default_rng(31)
    lens = [int(v) for v in rng.integers(0, 71, size=1100)]
    x = kda_inputs.make_random("t", lens, 1, seed=31, state_std=0.1)
    o_ref, s_ref = oracle.fwd_inputs(x)
    o, s = run_gpu(x, "chunked")
    check(o, s, o_ref, s_ref, "many documents")


@pytest.mark.parametrize("lb", [0.0, -0.5, -2.0])
def test_lower_bounds(cuda_device, lb):
    x = kda_inputs.make_random("t", [300, 77], 3, seed=22, state_std=0.1, lower_bound=lb)
    o_ref, s_ref = oracle.fwd_inputs(x)
    check(*run_gpu(x), o_ref, s_ref, f"lb={lb}")


def test_saturated_gates_and_extreme_beta(cuda_device):
    x = kda_inputs.make_random("t", [256, 100], 2, seed=23, state_std=0.1)
    x.g[:, :128].fill_(60.0)            # log alpha = -5 on every channel (fastest decay)
    x.g[:, 128:200].fill_(-60.0)        # log alpha ~ 0 (no decay)
    x.beta[:, ::3].fill_(30.0)          # beta = 1
    x.beta[:, 1::3].fill_(-30.0)        # beta ~ 0
    o_ref, s_ref = oracle.fwd_inputs(x)
    check(*run_gpu(x), o_ref, s_ref, "saturated")


def test_extreme_gate_parameters(cuda_device):
    # A_log = -inf: exp(A_log) = 0 and log alpha = lb / 2 on every channel; A_log = -100: exp(A_log)
    # is below float range on the GPU and the gate is sigmoid(0) there too; A_log = 30: every gate
    # saturates at log alpha = lb or 0; dt_bias = +inf / -inf on some channels of head 3: log alpha
    # = lb / 0 there.  Document lengths leave partial last chunks, whose masked rows must still get
    # alpha = 1 whatever the gate parameters are.
    x = kda_inputs.make_random("t", [100, 37, 200], 4, seed=31, state_std=0.1)
    x.A_log[0] = float("-inf")
    x.A_log[1] = -100.0
    x.A_log[2] = 30.0
    x.dt_bias[3, :16] = float("inf")
    x.dt_bias[3, 16:24] = float("-inf")
    o_ref, s_ref = oracle.fwd_inputs(x)
    assert np.isfinite(o_ref).all() and np.isfinite(s_ref).all()
    for impl in IMPLS:
        check(*run_gpu(x, impl), o_ref, s_ref, f"extreme A_log/{impl}")


def test_transposed_state_and_aliasing(cuda_device):
    x = kda_inputs.make_random("t", [150, 64], 2, seed=24, state_std=0.3)
    o_ref, s_ref = oracle.fwd_inputs(x, state_transposed=True)
    for impl in IMPLS:
        check(*run_gpu(x, impl, state_transposed=True), o_ref, s_ref, f"transposed/{impl}")
    o_ref, s_ref = oracle.fwd_inputs(x)
    for impl in IMPLS:
        check(*run_gpu(x, impl, alias=True), o_ref, s_ref, f"alias/{impl}")


def test_batch_mode(cuda_device):
    x = kda_inputs.make_random("t", None, 4, seed=25, varlen=False, batch=3, seqlen=190, state_std=0.1)
    o_ref, s_ref = oracle.fwd_inputs(x)
    for impl in IMPLS:
        check(*run_gpu(x, impl), o_ref, s_ref, f"batch/{impl}")


def test_varlen_matches_independent_documents_on_gpu(cuda_device):
    x = kda_inputs.make_random("t", [70, 129, 5], 2, seed=26, state_std=0.1)
    o, s = run_gpu(x)
    cu = x.cu_seqlens.tolist()
    for n in range(3):
        a, b = cu[n], cu[n + 1]
        xn = kda_inputs.KDAInputs("doc", x.q[:, a:b].contiguous(), x.k[:, a:b].contiguous(),
                                  x.v[:, a:b].contiguous(), x.g[:, a:b].contiguous(),
                                  x.beta[:, a:b].contiguous(), x.A_log, x.dt_bias, x.lower_bound, x.scale,
                                  x.initial_state[n:n + 1].contiguous(),
                                  torch.tensor([0, b - a], dtype=torch.int32))
        on, sn = run_gpu(xn)
        np.testing.assert_allclose(o[:, a:b], on, rtol=0, atol=1e-6)
        np.testing.assert_allclose(s[n:n + 1], sn, rtol=0, atol=1e-6)


def test_split_resume_on_gpu(cuda_device):
    x = kda_inputs.make_random("t", [400], 2, seed=27, state_std=0.1)
    o_ref, s_ref = oracle.fwd_inputs(x)
    t1 = 173
    part = lambda a, b, s0: kda_inputs.KDAInputs(
        "p", x.q[:, a:b].contiguous(), x.k[:, a:b].contiguous(), x.v[:, a:b].contiguous(),
        x.g[:, a:b].contiguous(), x.beta[:, a:b].contiguous(), x.A_log, x.dt_bias, x.lower_bound,
        x.scale, s0, torch.tensor([0, b - a], dtype=torch.int32))
    oa, sa = run_gpu(part(0, t1, x.initial_state))
    ob, sb = run_gpu(part(t1, 400, torch.from_numpy(sa).float()))
    check(np.concatenate([oa, ob], axis=1), sb, o_ref, s_ref, "split-resume")


@pytest.mark.parametrize("layout", ["varlen", "two stages"])
def test_chunked_is_deterministic(cuda_device, layout):
    """Bitwise-equal results over repeated calls: items are taken from a counter in whatever order
    the CTAs reach it, and the two-stage schedule overlaps launches, but no result depends on it."""
    if layout == "varlen":
        x = kda_inputs.make_workload("varlen")
    else:
        x = kda_inputs.make_random("t", [1000, 0, 2048, 77, 1, 3000, 0], 4, seed=32, state_std=0.1)
    o1, s1 = run_gpu(x)
    for _ in range(4):
        o2, s2 = run_gpu(x)
        np.testing.assert_array_equal(o1, o2)
        np.testing.assert_array_equal(s1, s2)


def test_device_wait_timeout_is_reported(cuda_device):
    """A bounded device wait on a barrier that nothing completes runs out, records
    KDA_ERR_DEVICE_TIMEOUT in the status word (read and cleared once) and leaves the context
    usable: a valid forward on the same workspace follows."""
    x = kda_inputs.make_workload("tail")
    ws = kda.new_workspace(x.total_tokens, x.num_heads, x.num_seqs, cuda_device)
    kda.selftest_wait_timeout(ws, limit_us=2000)
    assert kda.read_device_status(ws) == 5  # KDA_ERR_DEVICE_TIMEOUT
    assert kda.read_device_status(ws) == 0  # cleared by the read
    o_ref, s_ref = oracle.fwd_inputs(x)
    check(*run_gpu(x), o_ref, s_ref, "valid call after a time-out")


@pytest.mark.parametrize("bad", [[0, 200, 100, 350], [0, 100, 300, 100000], [0, 100, 300, 340],
                                 [5, 100, 300, 350], [0, -20, 300, 350]])
def test_malformed_cu_seqlens_reported_on_device(cuda_device, bad):
    """Offsets that do not tile the T tokens in order are caught on the device: the call records
    KDA_ERR_INVALID_ARGUMENT, touches no token outside [0, T), leaves out unwritten and hands the
    initial state through; the same workspace then serves a valid call."""
    x = kda_inputs.make_random("t", [100, 200, 50], 2, seed=40, state_std=0.1).to(cuda_device)
    N, H = 3, 2
    cu_bad = torch.tensor(bad, dtype=torch.int32, device=cuda_device)
    ws = kda.new_workspace(x.total_tokens, H, N, cuda_device)
    for fn in (kda.fwd, kda.fwd_recurrent):
        out = torch.full_like(x.v, float("nan"))
        fin = torch.full((N, H, 128, 128), float("nan"), device=cuda_device)
        fn(x.q, x.k, x.v, x.g, x.beta, x.scale, out, ws, x.A_log, x.dt_bias, x.lower_bound,
           x.initial_state, fin, cu_bad)
        assert kda.read_device_status(ws) == 1  # KDA_ERR_INVALID_ARGUMENT
        # every document is treated as empty, on both paths
        assert torch.isnan(out).all()
        assert torch.equal(fin, x.initial_state)
    o_ref, s_ref = oracle.fwd_inputs(x.to("cpu"))
    check(*run_gpu(x.to("cpu")), o_ref, s_ref, "valid call after a malformed one")


def test_chunk_kda_convenience(cuda_device):
    x = kda_inputs.make_workload("usage").to(cuda_device)
    out, final = kda.chunk_kda(x.q, x.k, x.v, x.g, x.beta, scale=x.scale, A_log=x.A_log,
                               dt_bias=x.dt_bias, lower_bound=x.lower_bound)
    assert final is None
    o_ref, _ = oracle.fwd_inputs(x.to("cpu"))
    check(out.float().cpu().double().numpy(), None, o_ref, None, "chunk_kda")
