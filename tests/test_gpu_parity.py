"""GPU parity of the StagQ GEMV against the CPU oracle (needs a B200).

Small cases: the GPU reads a stream packed from the ORACLE's fields, and y is
compared element by element with the oracle's fp64 GEMV. Full Llama-3.1-8B
shapes: the library encoder feeds the GPU (as in bench.py), the oracle encodes
the same weights independently, and sampled rows are compared (fields and y).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import quantized_gemv_stagq_b200 as Q
from oracle import stagq as O
from quantized_gemv_stagq_b200 import synth
from tests.helpers import check_close, fields_equal, lib_columns, n1_kernels, nb_kernels, to_lib_fields

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _needs_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    Q.lib()


def _load(F):
    return Q.stagq_load(Q.stagq_pack(to_lib_fields(F)), 0)


def _gemv(m, bits, x_np, f32=True, kernel=0):
    x = torch.from_numpy(np.ascontiguousarray(x_np)).cuda()
    n = x.shape[0]
    y = torch.empty(n, m.out, dtype=torch.float32 if f32 else torch.float16, device="cuda")
    Q.stagq_gemv_ex(m, bits, x, y, n=n, flags=(Q.STAGQ_Y_F32 if f32 else 0) | kernel)
    torch.cuda.synchronize()
    return y.cpu().numpy()


SMALL = [
    # out, in, group, n_planes, density, pair mode, seed
    (512, 512, 128, 2, 0.005, "search", 1),     # the tiny workload
    (96, 2048, 64, 4, 0.01, "fast", 2),         # deep stream, p2..p6
    (37, 640, 128, 2, 0.005, "fast", 3),        # fewer rows than SMs; ragged K (10 chunks)
    (300, 5120, 128, 2, 0.001, "fast", 4),      # K = 2.5 warp tiles
    (1, 4096, 128, 2, 0.01, "fast", 5),         # a single row
    (160, 1024, 64, 3, 0.0, "fast", 6),         # no side record
    (64, 768, 128, 2, 1.0, "fast", 7),          # everything held out
    (200, 4096, 128, 1, 0.02, "fast", 8),       # one plane
    (296, 4096, 128, 2, 0.6, "fast", 9),        # > 2048 record entries per stage (overflow path)
    (300, 32768, 128, 4, 0.005, "fast", 10),    # widest K: 16 K-warps, one-row stages at p6
    # groups of 16 / 32 (the paper's encoder settings; its kernel runs at 32): 2 or 4 pairs per chunk
    (512, 512, 32, 2, 0.005, "fast", 11),       # the tiny workload at g = 32 (0.25 bpw pair)
    (96, 2048, 16, 4, 0.01, "fast", 12),        # g = 16, deep stream, p2..p6
    (37, 640, 32, 3, 0.02, "fast", 13),         # g = 32, ragged K, fewer rows than SMs
    (300, 5120, 16, 2, 0.005, "fast", 14),      # g = 16, K = 2.5 warp tiles
    (64, 768, 16, 2, 1.0, "fast", 15),          # g = 16, everything held out
    (48, 256, 16, 2, 0.02, "search", 16),       # g = 16, searched pairs
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}g{c[2]}p{c[3]}d{c[4]}")
def test_decoded_levels_bit_exact(case):
    out, inp, g, npl, dens, mode, seed = case
    F = O.encode(synth.weights(out, inp, seed), g, npl, dens, mode)
    m = _load(F)
    u = torch.empty(out, inp, dtype=torch.uint8, device="cuda")
    for M in range(2, 3 + npl):
        Q.stagq_decode_levels(m, M, u)
        torch.cuda.synchronize()
        assert np.array_equal(u.cpu().numpy(), O.decode_levels(F, M)), f"p{M}"
    m.free()


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}g{c[2]}p{c[3]}d{c[4]}")
def test_gemv_matches_oracle(case):
    out, inp, g, npl, dens, mode, seed = case
    F = O.encode(synth.weights(out, inp, seed), g, npl, dens, mode)
    m = _load(F)
    x = synth.activations(1, inp, seed + 100)
    for M in range(2, 3 + npl):
        ref = O.gemv(F, M, x)
        for kern in n1_kernels(inp):  # both n = 1 kernels
            check_close(_gemv(m, M, x, f32=True, kernel=kern), ref, f"fp32 y p{M} kernel {kern}")
            check_close(_gemv(m, M, x, f32=False, kernel=kern).astype(np.float64), ref, f"fp16 y p{M} kernel {kern}")
    Q.stagq_check(m)
    m.free()


@pytest.mark.parametrize("case", SMALL, ids=lambda c: f"{c[0]}x{c[1]}g{c[2]}p{c[3]}d{c[4]}")
def test_batched_gemv_matches_oracle(case):
    """n = 2..4 activation vectors in one launch (the weights are read once):
    every column against the oracle, at every precision of the stream."""
    out, inp, g, npl, dens, mode, seed = case
    F = O.encode(synth.weights(out, inp, seed), g, npl, dens, mode)
    m = _load(F)
    for n in (2, 3, 4):
        x = synth.activations(n, inp, seed + 200 + n)
        for M in range(2, 3 + npl):
            ref = O.gemv(F, M, x)
            for kern in (0,) + nb_kernels(inp, g):  # the default and every kernel that serves n > 1
                got = _gemv(m, M, x, f32=True, kernel=kern)
                for j in range(n):
                    check_close(got[j], ref[j], f"n{n} col{j} p{M} kernel {kern}")
                got16 = _gemv(m, M, x, f32=False, kernel=kern).astype(np.float64)
                check_close(got16[n - 1], ref[n - 1], f"n{n} fp16 last col p{M} kernel {kern}")
            # each column agrees with the single-vector launch of that column
            one = _gemv(m, M, x[n - 1:n], f32=True)
            check_close(got[n - 1:n], one, f"n{n} last col vs n1 p{M}")
    Q.stagq_check(m)
    m.free()


def test_gemv_activation_edge_cases():
    out, inp = 256, 2048
    F = O.encode(synth.weights(out, inp, 11), 128, 2, 0.005, "fast")
    m = _load(F)
    rng = np.random.default_rng(0)
    xs = {
        "zeros": np.zeros((1, inp), np.float16),
        "one_hot": np.eye(1, inp, 1234, dtype=np.float16),
        "large": (rng.standard_normal((1, inp)) * 300).astype(np.float16),
        "tiny": (rng.standard_normal((1, inp)) * 1e-4).astype(np.float16),
        "mixed_scale": np.concatenate([rng.standard_normal(inp // 2) * 1e3,
                                       rng.standard_normal(inp // 2) * 1e-3]).astype(np.float16)[None],
    }
    for name, x in xs.items():
        for M in (2, 3, 4):
            y = _gemv(m, M, x)
            ref = O.gemv(F, M, x)
            if name == "zeros":
                assert not np.any(y), name
            else:
                check_close(y, ref, f"{name} p{M}")
    m.free()


def test_gemv_is_deterministic_and_reentrant():
    F = O.encode(synth.weights(1024, 4096, 21), 128, 2, 0.005, "fast")
    m = _load(F)
    x = torch.from_numpy(synth.activations(1, 4096, 22)).cuda()
    ys = []
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for kern in (Q.STAGQ_KERNEL_GENERAL, Q.STAGQ_KERNEL_SINGLE):
        ys = []
        for st in (s1, s2, s1):
            y = torch.empty(1, 1024, dtype=torch.float32, device="cuda")
            with torch.cuda.stream(st):
                Q.stagq_gemv_ex(m, 3, x, y, flags=Q.STAGQ_Y_F32 | kern, stream=st)
            ys.append(y)
        torch.cuda.synchronize()
        assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2]), f"kernel {kern}"
    m.free()


def test_host_buffer_call_and_file_round_trip(tmp_path):
    F = O.encode(synth.weights(384, 1024, 31), 128, 2, 0.005, "fast")
    S = Q.stagq_pack(to_lib_fields(F))
    m = Q.stagq_load(S, 0)
    path = str(tmp_path / "w.stagq")
    Q.stagq_save(S, path)
    mf = Q.stagq_load_file(path, 0)
    x = synth.activations(1, 1024, 32)
    for M in (2, 3, 4):
        y_dev = _gemv(m, M, x, f32=False)
        y_file = _gemv(mf, M, x, f32=False)
        y_host = np.empty((1, 384), np.float16)
        Q.stagq_gemv_host(m, M, x, y_host)
        assert np.array_equal(y_dev.view(np.uint16), y_file.view(np.uint16))
        assert np.array_equal(y_dev.view(np.uint16), y_host.view(np.uint16))
        assert Q.stagq_bytes(m, M) == O.model_bytes(384, 1024, 128, F.nnz, M)
    m.free()
    mf.free()


def test_bad_calls_return_errors():
    F = O.encode(synth.weights(64, 512, 41), 128, 2, 0.005, "fast")
    m = _load(F)
    x = torch.zeros(1, 512, dtype=torch.float16, device="cuda")
    y = torch.zeros(1, 64, dtype=torch.float16, device="cuda")
    for bits in (1, 5, 7):
        with pytest.raises(Q.StagqError) as e:
            Q.stagq_gemv(m, bits, x, y)
        assert e.value.status == 1
    with pytest.raises(Q.StagqError):
        Q.stagq_gemv_n(m, 2, x, 0, y)
    with pytest.raises(Q.StagqError):
        Q.stagq_gemv_ex(m, 2, x, y, flags=8)
    with pytest.raises(Q.StagqError):  # both kernels forced
        Q.stagq_gemv_ex(m, 2, x, y, flags=Q.STAGQ_KERNEL_GENERAL | Q.STAGQ_KERNEL_SINGLE)
    x4 = torch.zeros(4, 512, dtype=torch.float16, device="cuda")
    y4 = torch.zeros(4, 64, dtype=torch.float16, device="cuda")
    m32 = _load(O.encode(synth.weights(64, 512, 42), 32, 2, 0.005, "fast"))
    with pytest.raises(Q.StagqError):  # the single-vector kernel with n > 1 and groups below 64
        Q.stagq_gemv_ex(m32, 2, x4, y4, n=4, flags=Q.STAGQ_KERNEL_SINGLE)
    Q.stagq_gemv_ex(m, 2, x4, y4, n=4, flags=Q.STAGQ_KERNEL_SINGLE)  # groups of 128: planned
    torch.cuda.synchronize()
    m32.free()
    m.free()


LLAMA = list(synth.LLAMA31_8B_LINEARS.items())
SAMPLE_ROWS = 48


def _sampled_rows_case(out, inp, group, n_planes, density, seed, bits_list, kernels, batch4=True, **guard):
    """Library encoder -> GPU (as the bench does); the oracle encodes the same
    weights itself on sampled rows; fields and y agree on those rows."""
    W = synth.weights(out, inp, seed=seed)
    P = Q.stagq_encode(W, group, n_planes, density, "fast", **guard)
    m = Q.stagq_load(Q.stagq_pack(P), 0)
    rng = np.random.default_rng(out + inp)
    rows = np.unique(np.concatenate([[0, out - 1], rng.choice(out, SAMPLE_ROWS, replace=False)]))
    F = O.encode(W, group, n_planes, density, "fast", rows=rows, **guard)
    Psub = Q.Fields(F.out, inp, group, n_planes, P.q[rows], P.planes[:, rows], P.pair_idx[rows],
                    P.cb_log2s, P.cb_lo_over_s,
                    np.concatenate([[0], np.cumsum(np.diff(P.row_ptr)[rows])]).astype(np.int32),
                    np.concatenate([P.col[P.row_ptr[r]:P.row_ptr[r + 1]] for r in rows]),
                    np.concatenate([P.val[P.row_ptr[r]:P.row_ptr[r + 1]] for r in rows]))
    eq = fields_equal(F, Psub)
    assert all(eq.values()), eq
    x = synth.activations(4, inp, seed=7)
    for M in bits_list:
        ref1 = O.gemv(F, M, x[:1])[0]
        for kern in kernels:
            y = _gemv(m, M, x[:1], f32=False, kernel=kern)[0]
            check_close(y[rows].astype(np.float64), ref1, f"{out}x{inp} p{M} kernel {kern}")
            assert np.all(np.isfinite(y))
        if batch4:
            ref4 = O.gemv(F, M, x)
            for kern in (0,) + nb_kernels(inp, group):  # batch 4 in one launch
                y4 = _gemv(m, M, x, f32=False, kernel=kern)
                for j in range(4):
                    check_close(y4[j][rows].astype(np.float64), ref4[j], f"{out}x{inp} p{M} n4 col{j} kernel {kern}")
    Q.stagq_check(m)
    m.free()




def _kernels():
    return (0, Q.STAGQ_KERNEL_GENERAL, Q.STAGQ_KERNEL_SINGLE)


@pytest.mark.parametrize("name,shape", [(n, s) for n, s in LLAMA if n in ("q_proj", "k_proj", "gate_proj", "down_proj")])
def test_full_size_llama_sampled_rows(name, shape):
    """The bench's workload and launch at full Llama-3.1-8B shapes."""
    out, inp = shape
    _sampled_rows_case(out, inp, 128, 2, 0.005, 1000 + out + inp, (2, 3, 4), _kernels())


OTHER = [("phi4." + k, v) for k, v in synth.PHI4_LINEARS.items()] + \
        [("olmo2." + k, v) for k, v in synth.OLMO2_7B_LINEARS.items()]


@pytest.mark.parametrize("name,shape", OTHER, ids=[n for n, _ in OTHER])
def test_full_size_phi4_olmo2_sampled_rows(name, shape):
    """The Phi-4 and OLMo-2-7B linears of the bench at full size, 2/3/4 bits."""
    out, inp = shape
    _sampled_rows_case(out, inp, 128, 2, 0.005, 2000 + out + inp, (2, 3, 4), (0,), batch4=False)


@pytest.mark.parametrize("group,density", [(64, 0.0), (128, 0.001), (64, 0.01), (32, 0.005), (16, 0.005)])
def test_full_size_sweep_sampled_rows(group, density):
    """The precision/structure sweep: base + 4 planes read at 2..6 bits."""
    _sampled_rows_case(14336, 4096, group, 4, density, 3000 + group, (2, 3, 4, 5, 6), _kernels(), batch4=False)


# ------------------------------------- side-record guards (Section 3.5, Appendix E)

GUARDED = [
    # out, in, group, n_planes, ratio T, post-grid guard, seed
    (512, 512, 32, 2, 4.0, True, 21),      # the tiny workload at the paper's g = 32
    (96, 2048, 64, 4, 4.0, True, 22),      # deep stream, p2..p6
    (37, 640, 128, 3, 2.0, True, 23),      # ragged K, fewer rows than SMs, lower T
    (300, 5120, 16, 2, 4.0, True, 24),     # g = 16, K = 2.5 warp tiles
    (1, 4096, 128, 2, 4.0, True, 25),      # a single row
    (200, 4096, 128, 1, 8.0, False, 26),   # pre-grid guard only
]


def _guarded_fields(case):
    out, inp, g, npl, T, post, seed = case
    W = synth.weights(out, inp, seed)
    W[0, 7] = np.float16(0.8)              # a dominant entry in row 0's first group
    return O.encode(W, g, npl, mode="fast", guard="ratio", ratio_T=T, post_guard=post)


@pytest.mark.parametrize("case", GUARDED, ids=lambda c: f"{c[0]}x{c[1]}g{c[2]}p{c[3]}T{c[4]}{'post' if c[5] else ''}")
def test_guarded_gemv_matches_oracle(case):
    """Pre-grid entries (P = recorded value) and post-grid entries (P = lo + s q
    + r, zero planes) through both n = 1 kernels and the batched launch."""
    F = _guarded_fields(case)
    assert F.nnz > 0 and F.post_flags.sum() == (F.out if case[5] else 0)
    m = _load(F)
    u = torch.empty(F.out, F.inp, dtype=torch.uint8, device="cuda")
    for M in range(2, 3 + F.n_planes):
        Q.stagq_decode_levels(m, M, u)
        torch.cuda.synchronize()
        assert np.array_equal(u.cpu().numpy(), O.decode_levels(F, M)), f"levels p{M}"
        x = synth.activations(4, F.inp, case[6] + M)
        ref = O.gemv(F, M, x)
        for kern in (Q.STAGQ_KERNEL_GENERAL, Q.STAGQ_KERNEL_SINGLE):
            check_close(_gemv(m, M, x[:1], kernel=kern)[0], ref[0], f"p{M} kernel {kern}")
        for n in (2, 4):
            got = _gemv(m, M, x[:n])
            for j in range(n):
                check_close(got[j], ref[j], f"p{M} n{n} col{j}")
    Q.stagq_check(m)
    m.free()


@pytest.mark.parametrize("name,shape,group", [("gate_proj", (14336, 4096), 32), ("down_proj", (4096, 14336), 128)])
def test_full_size_guarded_sampled_rows(name, shape, group):
    """Full Llama-3.1-8B shapes with the ratio guard (T = 4) and the post-grid
    guard, as the paper configures its feed-forward matrices (Table 6)."""
    out, inp = shape
    _sampled_rows_case(out, inp, group, 2, 0.0, 4000 + out + group, (2, 3, 4), _kernels(), batch4=True,
                       guard="ratio", ratio_T=4.0)


def test_appendix_e_codebooks_gemv_matches_oracle():
    """Lloyd-placed codebooks (Appendix E's rules win on groups of widely
    spread scales) through both n = 1 kernels and n = 4."""
    from tests.test_oracle_pins import _weights_with_spread_scales
    W = _weights_with_spread_scales(64, 1024, 9)
    F = O.encode(W, 32, 2, 0.005, "fast", codebooks="appendix_e")
    assert not np.array_equal(F.cb_log2s, O.encode(W, 32, 2, 0.005, "fast").cb_log2s)
    m = _load(F)
    x = synth.activations(4, 1024, 10)
    for M in (2, 3, 4):
        ref = O.gemv(F, M, x)
        for kern in (Q.STAGQ_KERNEL_GENERAL, Q.STAGQ_KERNEL_SINGLE):
            check_close(_gemv(m, M, x[:1], kernel=kern)[0], ref[0], f"p{M} kernel {kern}")
        got = _gemv(m, M, x)
        for j in range(4):
            check_close(got[j], ref[j], f"p{M} n4 col{j}")
    Q.stagq_check(m)
    m.free()


# ------------------------------- stacked handles (q/k/v or gate/up in one launch)

STACKED = [
    # member shapes (out) at a common in, group, n_planes, density, guards
    ((192, 64, 64), 1024, 128, 2, 0.005, None),
    ((96, 33, 160), 2048, 64, 4, 0.01, None),
    ((37, 100), 640, 32, 3, 0.02, None),
    ((64, 48, 80, 16), 1024, 128, 2, 0.0, "ratio"),   # pre- and post-grid guards, four members
]


def _stack_fields(case, seed0):
    outs, inp, g, npl, dens, guard = case
    Fs = []
    for j, out in enumerate(outs):
        W = synth.weights(out, inp, seed0 + j)
        if guard == "ratio":
            Fs.append(O.encode(W, g, npl, mode="fast", guard="ratio", ratio_T=4.0, post_guard=True))
        else:
            Fs.append(O.encode(W, g, npl, dens, "fast"))
    return Fs


@pytest.mark.parametrize("case", STACKED, ids=lambda c: f"{'+'.join(map(str, c[0]))}x{c[1]}g{c[2]}p{c[3]}")
def test_stacked_handle_matches_each_member(case):
    """Each member's rows of a stacked handle against the oracle's GEMV of that
    member alone (its own codebooks, pair bytes and side record), through both
    n = 1 kernels, n = 4, and the decoded levels bit-exact."""
    Fs = _stack_fields(case, 500)
    assert len({tuple(F.cb_log2s.view(np.uint16)) for F in Fs}) > 1   # the members' codebooks differ
    m = Q.stagq_load_stack([Q.stagq_pack(to_lib_fields(F)) for F in Fs], 0)
    assert m.out == sum(F.out for F in Fs)
    offs = np.concatenate([[0], np.cumsum([F.out for F in Fs])])
    u = torch.empty(m.out, m.inp, dtype=torch.uint8, device="cuda")
    x = synth.activations(4, m.inp, 77)
    for M in range(2, 3 + Fs[0].n_planes):
        Q.stagq_decode_levels(m, M, u)
        torch.cuda.synchronize()
        assert np.array_equal(u.cpu().numpy(), np.concatenate([O.decode_levels(F, M) for F in Fs])), f"levels p{M}"
        refs = [O.gemv(F, M, x) for F in Fs]
        for kern in (Q.STAGQ_KERNEL_GENERAL, Q.STAGQ_KERNEL_SINGLE):
            y = _gemv(m, M, x[:1], kernel=kern)[0]
            for j, F in enumerate(Fs):
                check_close(y[offs[j]:offs[j + 1]], refs[j][0], f"member {j} p{M} kernel {kern}")
        y4 = _gemv(m, M, x)
        for j, F in enumerate(Fs):
            for c in range(4):
                check_close(y4[c][offs[j]:offs[j + 1]], refs[j][c], f"member {j} p{M} n4 col{c}")
        # x read once, one row-pointer array for the whole stack
        assert Q.stagq_bytes(m, M) == sum(O.model_bytes(F.out, F.inp, F.group, F.nnz, M) for F in Fs) \
            - (len(Fs) - 1) * (2 * m.inp + 4)
    Q.stagq_check(m)
    m.free()


@pytest.mark.parametrize("name,members", [("qkv", ("q_proj", "k_proj", "v_proj")), ("gate_up", ("gate_proj", "up_proj"))])
def test_full_size_stacked_llama_sampled_rows(name, members):
    """The bench's stacked Llama-3.1-8B handles (q/k/v: 6144 x 4096, gate/up:
    28672 x 4096): library encoder per member, every member's sampled rows and
    first / last rows against the oracle's own encoding of that member."""
    shapes = [synth.LLAMA31_8B_LINEARS[n] for n in members]
    Ws = [synth.weights(o, i, seed=5000 + j) for j, (o, i) in enumerate(shapes)]
    Ps = [Q.stagq_encode(W, 128, 2, 0.005, "fast") for W in Ws]
    m = Q.stagq_load_stack([Q.stagq_pack(P) for P in Ps], 0)
    x = synth.activations(1, shapes[0][1], seed=8)
    rng = np.random.default_rng(9)
    off = 0
    ys = {M: {k: _gemv(m, M, x, f32=False, kernel=k)[0] for k in _kernels()} for M in (2, 3, 4)}
    for j, ((o, i), W) in enumerate(zip(shapes, Ws)):
        rows = np.unique(np.concatenate([[0, o - 1], rng.choice(o, 24, replace=False)]))
        F = O.encode(W, 128, 2, 0.005, "fast", rows=rows)
        assert np.array_equal(F.pair_idx, Ps[j].pair_idx[rows]) and np.array_equal(F.q, Ps[j].q[rows])
        for M in (2, 3, 4):
            ref = O.gemv(F, M, x)[0]
            for k, y in ys[M].items():
                check_close(y[off + rows].astype(np.float64), ref, f"{name} member {j} p{M} kernel {k}")
        off += o
    Q.stagq_check(m)
    m.free()


# ------------------------- run-time inverse activation scale (Appendix E)

def _in_scale(inp, seed):
    """1/a_c for AWQ-like channel scales a_c spread over [0.25, 4] (log-uniform)."""
    rng = np.random.default_rng(seed)
    return (2.0 ** rng.uniform(-2.0, 2.0, inp)).astype(np.float32)


def _gemv_scaled(m, bits, x_np, s_np, f32=True, kernel=0):
    x = torch.from_numpy(np.ascontiguousarray(x_np)).cuda()
    s = torch.from_numpy(np.ascontiguousarray(s_np)).cuda()
    n = x.shape[0]
    y = torch.empty(n, m.out, dtype=torch.float32 if f32 else torch.float16, device="cuda")
    Q.stagq_gemv_scaled(m, bits, x, s, y, n=n, flags=(Q.STAGQ_Y_F32 if f32 else 0) | kernel)
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("case", [SMALL[0], SMALL[1], SMALL[3], SMALL[10], SMALL[12]],
                         ids=lambda c: f"{c[0]}x{c[1]}g{c[2]}p{c[3]}d{c[4]}")
def test_scaled_gemv_matches_oracle(case):
    """y = W_hat (x * in_scale) against the oracle's gemv(in_scale=), through
    both n = 1 kernels and n = 4 in one launch."""
    out, inp, g, npl, dens, mode, seed = case
    F = O.encode(synth.weights(out, inp, seed), g, npl, dens, mode)
    m = _load(F)
    s = _in_scale(inp, seed + 1)
    x = synth.activations(4, inp, seed + 300)
    for M in range(2, 3 + npl):
        ref = O.gemv(F, M, x, in_scale=s)
        for kern in (Q.STAGQ_KERNEL_GENERAL, Q.STAGQ_KERNEL_SINGLE):
            check_close(_gemv_scaled(m, M, x[:1], s, kernel=kern)[0], ref[0], f"p{M} kernel {kern}")
        for kern in (0,) + nb_kernels(inp, g):
            got = _gemv_scaled(m, M, x, s, kernel=kern)
            for j in range(4):
                check_close(got[j], ref[j], f"p{M} n4 col{j} kernel {kern}")
        # a scale of ones is the unscaled GEMV
        ones = _gemv_scaled(m, M, x[:1], np.ones(inp, np.float32))
        check_close(ones[0], O.gemv(F, M, x[:1])[0], f"p{M} ones")
    Q.stagq_check(m)
    m.free()


def test_host_many_matches_single_host_calls():
    """stagq_gemv_host_many runs several GEMVs with host buffers and one
    synchronization; a repeated handle, three precisions and n = 1 and 4: each
    y equals the single-call host GEMV bit for bit, and equals the oracle."""
    Fa = O.encode(synth.weights(300, 1024, 51), 128, 2, 0.005, "fast")
    Fb = O.encode(synth.weights(96, 2048, 52), 64, 4, 0.01, "fast")
    ma, mb = _load(Fa), _load(Fb)
    xa1 = np.ascontiguousarray(synth.activations(1, 1024, 60))
    xb4 = np.ascontiguousarray(synth.activations(4, 2048, 61))
    xa4 = np.ascontiguousarray(synth.activations(4, 1024, 62))
    calls = [(ma, Fa, 2, xa1, 1), (mb, Fb, 5, xb4, 4), (ma, Fa, 4, xa4, 4), (ma, Fa, 3, xa1, 1)]
    ys = [np.zeros((n, m.out), np.float16) for m, _, _, _, n in calls]
    Q.stagq_gemv_host_many([c[0] for c in calls], [c[2] for c in calls], [c[3] for c in calls], ys,
                           ns=[c[4] for c in calls])
    for (m, F, b, x, n), y in zip(calls, ys):
        one = np.zeros((n, m.out), np.float16)
        Q.stagq_gemv_host(m, b, x, one, n=n)
        assert np.array_equal(y, one), f"p{b} n{n}"
        ref = O.gemv(F, b, x)
        for j in range(n):
            check_close(y[j].astype(np.float64), ref[j], f"p{b} n{n} col{j}")
    with pytest.raises(Q.StagqError):  # no GEMV
        Q.stagq_gemv_host_many([], [], [], [])
    with pytest.raises(Q.StagqError):  # bits outside the stream
        Q.stagq_gemv_host_many([ma], [7], [xa1], [ys[0]])
    with pytest.raises(Q.StagqError):  # n outside 1..4
        Q.stagq_gemv_host_many([ma], [2], [np.zeros((5, 1024), np.float16)], [np.zeros((5, 300), np.float16)], ns=[5])
    ma.free()
    mb.free()


def test_scaled_product_that_rounds_to_the_int16_limit():
    """x = 1 and s = 1 - 2^-17: every scaled product is 32767.75 after the
    chunk's power-of-two scale, which rounds to 2^15; the fixed-point value
    must stay inside int16 (a wrapped -2^15 would flip the sign of the chunk)."""
    out, inp = 64, 512
    F = O.encode(synth.weights(out, inp, 43), 128, 2, 0.005, "fast")
    m = _load(F)
    s = np.full(inp, 1.0 - 2.0 ** -17, np.float32)
    x = np.ones((4, inp), np.float16)
    for M in (2, 3, 4):
        ref = O.gemv(F, M, x, in_scale=s)
        for kern in (Q.STAGQ_KERNEL_GENERAL, Q.STAGQ_KERNEL_SINGLE):
            check_close(_gemv_scaled(m, M, x[:1], s, kernel=kern)[0], ref[0], f"p{M} kernel {kern}")
        for kern in (0, Q.STAGQ_KERNEL_GENERAL):
            got = _gemv_scaled(m, M, x, s, kernel=kern)
            for j in range(4):
                check_close(got[j], ref[j], f"p{M} n4 col{j} kernel {kern}")
    Q.stagq_check(m)
    m.free()


@pytest.mark.parametrize("name", ["gate_proj", "q_proj"])
def test_full_size_scaled_sampled_rows(name):
    """The Llama-3.1-8B gate (single-vector kernel) and q (general kernel)
    shapes with an inverse activation scale, n = 1 and 4, sampled rows."""
    out, inp = synth.LLAMA31_8B_LINEARS[name]
    W = synth.weights(out, inp, seed=6000 + out)
    P = Q.stagq_encode(W, 128, 2, 0.005, "fast")
    m = Q.stagq_load(Q.stagq_pack(P), 0)
    rows = np.unique(np.concatenate([[0, out - 1], np.random.default_rng(3).choice(out, 32, replace=False)]))
    F = O.encode(W, 128, 2, 0.005, "fast", rows=rows)
    s = _in_scale(inp, 5)
    x = synth.activations(4, inp, seed=6)
    for M in (2, 4):
        ref = O.gemv(F, M, x, in_scale=s)
        y1 = _gemv_scaled(m, M, x[:1], s, f32=False)[0]
        check_close(y1[rows].astype(np.float64), ref[0], f"{name} p{M} n1")
        y4 = _gemv_scaled(m, M, x, s, f32=False)
        for j in range(4):
            check_close(y4[j][rows].astype(np.float64), ref[j], f"{name} p{M} n4 col{j}")
    Q.stagq_check(m)
    m.free()


# --------------------------- the side record as the device holds it (Eq. 4)

def _expected_entries(F):
    """The oracle's side record per row: (column | post-grid flag << 15, fp16 bits)."""
    cols = lib_columns(F)
    vals = F.val.view(np.uint16)
    return [[(int(cols[e]), int(vals[e])) for e in range(F.row_ptr[r], F.row_ptr[r + 1])] for r in range(F.out)]


def _decode_cuts(out, lay, cut, cut1):
    """Rebuild each row's entries from the two device cuts (the layout of
    stagq_debug_side_record), independently of the loader's code."""
    rows_general = [[] for _ in range(out)]
    G, S, RG, KW, CR = lay["grid"], lay["stride"], lay["row_groups"], lay["k_slices"], lay["class_rows"]
    for b in range(G):
        blk = cut[b * S:(b + 1) * S]
        offs = blk[:4 * RG * KW * (CR + 1)].view(np.int32).reshape(RG, KW, CR + 1)
        ents = blk[lay["ent_off"]:].view(np.uint32)
        ra, rb = b * out // G, (b + 1) * out // G
        for rg in range(RG):
            nm = (rb - ra - rg + RG - 1) // RG if rb - ra > rg else 0
            for kw in range(KW):
                for mm in range(nm):
                    r = ra + rg + RG * mm
                    for e in ents[offs[rg, kw, mm]:offs[rg, kw, mm + 1]]:
                        rows_general[r].append((int(e & 0xFFFF), int(e >> 16)))
    rows_single = [[] for _ in range(out)]
    G1, S1 = lay["grid1"], lay["stride1"]
    for b in range(G1):
        blk = cut1[b * S1:(b + 1) * S1]
        ra, rb = b * out // G1, (b + 1) * out // G1
        offs = blk[:4 * (rb - ra + 1)].view(np.int32)
        ents = blk[lay["ent_off1"]:].view(np.uint32)
        for r in range(ra, rb):
            for e in ents[offs[r - ra]:offs[r - ra + 1]]:
                rows_single[r].append((int(e & 0xFFFF), int(e >> 16)))
    return rows_general, rows_single


@pytest.mark.parametrize("kind", ["tiny", "ragged", "dense60", "all", "guarded", "wideK", "stacked"])
def test_device_side_record_bit_exact(kind):
    """Both device cuts of the side record hold exactly the oracle's CSR:
    row, column, post-grid flag and fp16 value of every entry, in column
    order within a row."""
    if kind == "tiny":
        Fs = [O.encode(synth.weights(512, 512, 1), 128, 2, 0.005, "search")]
    elif kind == "ragged":
        Fs = [O.encode(synth.weights(37, 640, 3), 128, 2, 0.02, "fast")]
    elif kind == "dense60":
        Fs = [O.encode(synth.weights(296, 4096, 9), 128, 2, 0.6, "fast")]
    elif kind == "all":
        Fs = [O.encode(synth.weights(64, 768, 7), 16, 2, 1.0, "fast")]
    elif kind == "guarded":
        Fs = [_guarded_fields(GUARDED[0])]
    elif kind == "wideK":
        Fs = [O.encode(synth.weights(300, 32768, 10), 128, 4, 0.005, "fast")]
    else:
        Fs = _stack_fields(STACKED[3], 700)
    m = Q.stagq_load_stack([Q.stagq_pack(to_lib_fields(F)) for F in Fs], 0)
    lay, cut, cut1 = Q.stagq_debug_side_record(m)
    want = [row for F in Fs for row in _expected_entries(F)]
    assert sum(len(r) for r in want) == sum(F.nnz for F in Fs)
    got_general, got_single = _decode_cuts(m.out, lay, cut, cut1)
    assert got_general == want
    assert got_single == want
    m.free()


# ----------------------------- the bounded waits' give-up path (no GPU fault)

@pytest.mark.parametrize("kernel", ["general", "single"])
def test_wait_that_runs_out_is_reported_and_the_handle_recovers(kernel):
    """A launch whose bounded wait runs out (stagq_debug_stall: a barrier
    nothing completes, 20 us) lets its copies land, returns, and stagq_check
    reports STAGQ_ETIMEOUT; with the hook off the next call matches the
    oracle and stagq_check is clean."""
    flag = Q.STAGQ_KERNEL_GENERAL if kernel == "general" else Q.STAGQ_KERNEL_SINGLE
    F = O.encode(synth.weights(1024, 4096, 55), 128, 2, 0.005, "fast")
    m = _load(F)
    x = synth.activations(1, 4096, 56)
    Q.stagq_debug_stall(m, 20000)
    _gemv(m, 3, x, kernel=flag)
    with pytest.raises(Q.StagqError) as e:
        Q.stagq_check(m)
    assert e.value.status == 7                       # STAGQ_ETIMEOUT
    Q.stagq_debug_stall(m, 0)
    check_close(_gemv(m, 3, x, kernel=flag)[0], O.gemv(F, 3, x)[0], "after the stall")
    Q.stagq_check(m)                                  # the status word was cleared
    m.free()


# --------------------------------- full size, every row against the oracle

@pytest.mark.parametrize("name", ["gate_proj", "q_proj"])
def test_full_size_every_row(name):
    """Llama-3.1-8B gate (14336 x 4096, the single-vector kernel by default)
    and q (4096 x 4096, the general kernel by default): the oracle encodes the
    whole matrix (fast pair rule), the GPU reads the oracle's own fields, and
    every row of y is compared with the oracle's fp64 GEMV, through each n = 1
    kernel, at 2/3/4 bits; the CTA row partitions and per-CTA side-record cuts
    of the full grid are all exercised."""
    out, inp = synth.LLAMA31_8B_LINEARS[name]
    F = O.encode(synth.weights(out, inp, seed=7000 + out), 128, 2, 0.005, "fast")
    m = _load(F)
    x = synth.activations(1, inp, seed=7001)
    for M in (2, 3, 4):
        ref = O.gemv(F, M, x)[0]
        for kern in _kernels():
            check_close(_gemv(m, M, x, f32=True, kernel=kern)[0], ref, f"{name} p{M} kernel {kern} fp32")
        check_close(_gemv(m, M, x, f32=False)[0].astype(np.float64), ref, f"{name} p{M} fp16")
    Q.stagq_check(m)
    m.free()


def test_full_size_stacked_qkv_every_row():
    """The stacked q/k/v handle of the bench (6144 x 4096), every row of every
    member against the oracle's GEMV of that member."""
    Fs = [O.encode(synth.weights(*synth.LLAMA31_8B_LINEARS[n], seed=7100 + j), 128, 2, 0.005, "fast")
          for j, n in enumerate(("q_proj", "k_proj", "v_proj"))]
    m = Q.stagq_load_stack([Q.stagq_pack(to_lib_fields(F)) for F in Fs], 0)
    x = synth.activations(1, 4096, seed=7101)
    for M in (2, 4):
        for kern in _kernels():
            y = _gemv(m, M, x, kernel=kern)[0]
            off = 0
            for j, F in enumerate(Fs):
                check_close(y[off:off + F.out], O.gemv(F, M, x)[0], f"member {j} p{M} kernel {kern}")
                off += F.out
    Q.stagq_check(m)
    m.free()
