"""GPU vs oracle parity through the C ABI.

Bar (from the method's definition): ternary codes / packed bytes, α, x̃, β and
the int32 accumulators bit-exact; fp32 outputs within 1e-5 relative.  Inputs
are the seeded synthetic recipes; expected values come only from ``oracle``.
"""
import numpy as np
import pytest
import torch

import bitlinear_w1_a8_03_b200 as bl
import oracle
from bitlinear_w1_a8_03_b200 import synth
from tests.gpu_util import as_input, dev_f32, gpu_forward, gpu_quantize_weights, np_

pytestmark = pytest.mark.gpu

Y_RTOL = 1e-5


def assert_y_close(y, y_ref):
    err = np.abs(y.astype(np.float64) - y_ref.astype(np.float64))
    bound = Y_RTOL * np.abs(y_ref.astype(np.float64)) + 1e-37
    assert np.all(err <= bound), f"max rel err {np.max(err / (np.abs(y_ref) + 1e-37)):.3g}"


def check_weights(W_f32, dtype):
    Wd, Wo = as_input(W_f32, dtype)
    packed, alpha = gpu_quantize_weights(Wd)
    p_ref, a_ref, codes = oracle.quantize_weights(Wo)
    assert np_(alpha)[0] == a_ref, (np_(alpha)[0], a_ref)
    assert np.array_equal(np_(packed), p_ref)
    return packed, alpha, codes, a_ref


def check_forward(x_f32, dtype, packed, alpha, codes, a_ref, bias=None):
    N = codes.shape[0]
    xd, xo = as_input(x_f32, dtype)
    bd = None if bias is None else dev_f32(bias)
    xq, beta, acc, y = gpu_forward(xd, packed, alpha, N, bias=bd)
    xq_r, beta_r, acc_r, y_r = oracle.forward(xo, codes, a_ref, bias=bias, threads=8)
    assert np.array_equal(np_(xq), xq_r)
    assert np.array_equal(np_(beta), beta_r)
    assert np.array_equal(np_(acc), acc_r)
    assert_y_close(np_(y), y_r)
    return np_(y), y_r


# ---------------------------------------------------------------- pages' examples
def test_worked_example_on_gpu(golden):
    g = golden("worked_example.txt")
    t = golden("rounding_ties.txt")
    W = np.array([g["W"]], dtype=np.float32)
    packed, alpha, codes, a_ref = check_weights(W, "f32")
    assert codes.ravel().tolist() == [1, 0, 0, -1]
    assert np_(packed)[0, :4].tolist() == [0x56, 0x55, 0x55, 0x54]
    x = np.array([t["x2"]], dtype=np.float32)
    xd, _ = as_input(x, "f32")
    xq, beta, acc, y = gpu_forward(xd, packed, alpha, 1)
    assert np_(acc).tolist() == [[254]]
    assert np_(xq).ravel().tolist() == [127, 64, -64, -127]


def test_rounding_ties_on_gpu(golden):
    t = golden("rounding_ties.txt")
    W = np.array([t["W"]], dtype=np.float32)
    packed, alpha, codes, a_ref = check_weights(W, "f32")
    assert np_(alpha)[0] == 0.5
    assert codes.ravel().tolist() == [0, 1, 0, -1]
    xd, _ = as_input(np.array([t["x"]], dtype=np.float32), "f32")
    xq, beta, acc, y = gpu_forward(xd, packed, alpha, 1)
    assert np_(xq).ravel().tolist() == [127, 2, -2, 0]


# ---------------------------------------------------------------- tiny config
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tiny_config_bitexact(dtype):
    """M=1, K=N=256, W ~ N(0, 0.02), x ~ N(0, 1), seed 0."""
    W = synth.weights(0, 256, 256, 0.02)
    x = synth.activations(0, 1, 256)
    packed, alpha, codes, a_ref = check_weights(W, dtype)
    y, y_r = check_forward(x, dtype, packed, alpha, codes, a_ref)
    assert np.array_equal(y, y_r)  # the same scalar arithmetic on both sides: 0 ulp
    assert abs(float(np.mean(codes == 0)) - 0.31) < 0.02


# ---------------------------------------------------------------- edge shapes
@pytest.mark.parametrize("K", [1, 3, 4, 5, 16, 17, 48, 64, 65, 260, 1000, 4096 + 16])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 65])
def test_edge_shapes(M, K):
    N = 33
    seed = 100 + 7 * K + M
    W = synth.weights(seed, N, K, 0.02)
    x = synth.activations(seed, M, K, outliers=True)
    bias = synth.activations(seed + 1, 1, N)[0]
    packed, alpha, codes, a_ref = check_weights(W, "f32")
    check_forward(x, "bf16", packed, alpha, codes, a_ref, bias=bias)


@pytest.mark.parametrize("N", [1, 7, 8, 9, 1000])
def test_row_counts(N):
    K = 320
    W = synth.weights(N, N, K, 0.02)
    x = synth.activations(N, 4, K)
    packed, alpha, codes, a_ref = check_weights(W, "bf16")
    check_forward(x, "f32", packed, alpha, codes, a_ref)


def test_misaligned_activation_rows_use_generic_path():
    """x̃ at an odd address: the fast kernel needs 16-byte rows, so the generic
    kernel runs; results must be identical."""
    K, N, M = 128, 40, 3
    W = synth.weights(1, N, K, 0.02)
    x = synth.activations(1, M, K)
    packed, alpha, codes, a_ref = check_weights(W, "f32")
    import bitlinear_w1_a8_03_b200 as bl
    xd, xo = as_input(x, "f32")
    buf = torch.empty(M * K + 1, dtype=torch.int8, device="cuda")
    xq = buf[1:].view(M, K)
    beta = torch.empty(M, dtype=torch.float32, device="cuda")
    bl.bitlinear_quantize_act(xd, x_q=xq, beta=beta)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = bl.bitlinear_forward(xq, beta, packed, alpha, N, acc_out=acc)
    xq_r, beta_r, acc_r, y_r = oracle.forward(xo, codes, a_ref)
    assert np.array_equal(np_(xq), xq_r) and np.array_equal(np_(acc), acc_r)
    assert_y_close(np_(y), y_r)


# ---------------------------------------------------------------- degenerate inputs
def test_degenerate_inputs():
    K, N = 192, 24
    # all-zero weights: α = 0 and every code is the zero code
    Wz = np.zeros((N, K), dtype=np.float32)
    packed, alpha, codes, a_ref = check_weights(Wz, "f32")
    assert np_(alpha)[0] == 0.0 and np.all(np_(packed) == 0x55)
    # constant weights: every code is +1
    Wc = np.full((N, K), 0.0123, dtype=np.float32)
    packed, alpha, codes, a_ref = check_weights(Wc, "f32")
    assert np.all(codes == 1)
    # a zero token, a single-spike token and a token with ties
    x = np.zeros((3, K), dtype=np.float32)
    x[1, 5] = -7.0
    x[2, :4] = [127, 2.5, -2.5, 0]
    y, _ = check_forward(x, "f32", packed, alpha, codes, a_ref)
    assert np.all(y[0] == 0.0)


def test_alpha_underflow_and_denormals():
    """A mean that underflows to α = 0 with nonzero weights: W/α = ±inf → ±1,
    0/0 → zero code; and weights spanning many exponents."""
    K, N = 64, 4
    W = np.zeros((N, K), dtype=np.float32)
    W[0, 0] = np.float32(1e-45)
    W[1, 3] = -np.float32(1e-45)
    packed, alpha, codes, a_ref = check_weights(W, "f32")
    assert a_ref == 0.0 and codes[0, 0] == 1 and codes[1, 3] == -1 and codes[2, 0] == 0
    rng = np.random.default_rng(4)
    W = (np.sign(rng.standard_normal((N, K))) * np.exp2(rng.uniform(-140, 60, (N, K)))).astype(np.float32)
    check_weights(W, "f32")


# ---------------------------------------------------------------- grouped launches
def test_grouped_equals_single():
    import bitlinear_w1_a8_03_b200 as bl
    shapes = [(1, 256, 96), (3, 64, 40), (2, 1024, 300), (1, 4096, 512)]
    problems, refs = [], []
    xs, outs = [], []
    for i, (M, K, N) in enumerate(shapes):
        W = synth.weights(50 + i, N, K, 0.02)
        x = synth.activations(50 + i, M, K, outliers=True)
        packed, alpha, codes, a_ref = check_weights(W, "bf16")
        xd, xo = as_input(x, "bf16")
        xs.append(xd)
        outs.append((torch.empty((M, K), dtype=torch.int8, device="cuda"),
                     torch.empty(M, dtype=torch.float32, device="cuda")))
        problems.append(dict(x_q=outs[-1][0], beta=outs[-1][1], W_packed=packed, alpha=alpha, N=N,
                             y=torch.empty((M, N), dtype=torch.float32, device="cuda"),
                             acc_out=torch.empty((M, N), dtype=torch.int32, device="cuda")))
        refs.append(oracle.forward(xo, codes, a_ref))
    bl.bitlinear_quantize_act_grouped(xs, outs)
    bl.bitlinear_forward_grouped(problems)
    for p, (xq_r, beta_r, acc_r, y_r) in zip(problems, refs):
        assert np.array_equal(np_(p["x_q"]), xq_r)
        assert np.array_equal(np_(p["beta"]), beta_r)
        assert np.array_equal(np_(p["acc_out"]), acc_r)
        assert_y_close(np_(p["y"]), y_r)


# ---------------------------------------------------------------- guard bytes
def test_outputs_stay_in_bounds():
    """Canaries around every output buffer are untouched (no compute-sanitizer
    on this pool, so out-of-bounds writes are checked this way)."""
    import bitlinear_w1_a8_03_b200 as bl
    M, K, N = 5, 200, 37
    G = 256
    W = synth.weights(8, N, K, 0.02)
    x = synth.activations(8, M, K)
    Wd, _ = as_input(W, "f32")
    xd, _ = as_input(x, "f32")
    rb = bl.packed_row_bytes(K)

    def guarded(n, dtype):
        t = torch.full((n + 2 * G,), 0x5A if dtype == torch.uint8 else 0, dtype=dtype, device="cuda")
        if dtype != torch.uint8:
            t.view(torch.uint8).fill_(0x5A)
        return t

    pk = guarded(N * rb, torch.uint8)
    al = guarded(1, torch.float32)
    xq = guarded(M * K, torch.int8)
    be = guarded(M, torch.float32)
    y = guarded(M * N, torch.float32)
    ac = guarded(M * N, torch.int32)
    bl.bitlinear_quantize_weights(Wd, W_packed=pk[G:G + N * rb].view(N, rb), alpha=al[G:G + 1])
    bl.bitlinear_quantize_act(xd, x_q=xq[G:G + M * K].view(M, K), beta=be[G:G + M])
    bl.bitlinear_forward(xq[G:G + M * K].view(M, K), be[G:G + M], pk[G:G + N * rb].view(N, rb), al[G:G + 1], N,
                         y=y[G:G + M * N].view(M, N), acc_out=ac[G:G + M * N].view(M, N))
    torch.cuda.synchronize()
    for t, n in ((pk, N * rb), (al, 1), (xq, M * K), (be, M), (y, M * N), (ac, M * N)):
        raw = np_(t.view(torch.uint8))
        es = t.element_size()
        assert np.all(raw[: G * es] == 0x5A) and np.all(raw[(G + n) * es:] == 0x5A)


# ---------------------------------------------------------------- fused linear (PDL) path
@pytest.mark.parametrize("M,K,N", [(1, 4096, 300), (2, 1024, 77), (3, 512, 64), (5, 4096 + 16, 40), (1, 100, 9)])
def test_linear_matches_oracle(M, K, N):
    import bitlinear_w1_a8_03_b200 as bl
    W = synth.weights(K + N, N, K, 0.02)
    x = synth.activations(K + M, M, K, outliers=True)
    bias = synth.activations(7, 1, N)[0]
    packed, alpha, codes, a_ref = check_weights(W, "f32")
    xd, xo = as_input(x, "bf16")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    beta = torch.empty(M, dtype=torch.float32, device="cuda")
    y = bl.bitlinear_linear(xd, packed, alpha, N, bias=dev_f32(bias), x_q=xq, beta=beta, acc_out=acc)
    xq_r, beta_r, acc_r, y_r = oracle.forward(xo, codes, a_ref, bias=bias)
    assert np.array_equal(np_(xq), xq_r) and np.array_equal(np_(beta), beta_r)
    assert np.array_equal(np_(acc), acc_r)
    assert_y_close(np_(y), y_r)


@pytest.mark.parametrize("flags", [0, 1])
def test_linear_grouped_back_to_back_inputs_change(flags):
    """Steps with different inputs on the same buffers, queued without any
    host sync: each product must see its own step's x̃ (the weight stream
    starts before the quantisation kernel finishes)."""
    import bitlinear_w1_a8_03_b200 as bl
    shapes = [(4096, 4096), (4096, 1000), (1024, 512)]
    Ws = [synth.weights(70 + i, N, K, 0.02) for i, (K, N) in enumerate(shapes)]
    quant = [check_weights(W, "f32") for W in Ws]
    x_dev = [torch.empty((1, K), dtype=torch.bfloat16, device="cuda") for K, _ in shapes]
    xq = [torch.empty((1, K), dtype=torch.int8, device="cuda") for K, _ in shapes]
    beta = [torch.empty(1, dtype=torch.float32, device="cuda") for _ in shapes]
    steps = 4
    ys = [[torch.empty((1, N), dtype=torch.float32, device="cuda") for _, N in shapes] for _ in range(steps)]
    xo_all = []
    for t in range(steps):
        xo_step = []
        for i, (K, N) in enumerate(shapes):
            xd, xo = as_input(synth.activations(900 + 10 * t + i, 1, K, outliers=True), "bf16")
            x_dev[i].copy_(xd, non_blocking=True)
            xo_step.append(xo)
        xo_all.append(xo_step)
        probs = [dict(x=x_dev[i], x_q=xq[i], beta=beta[i], W_packed=quant[i][0], alpha=quant[i][1], N=N, y=ys[t][i])
                 for i, (K, N) in enumerate(shapes)]
        bl.bitlinear_linear_grouped(probs, flags=flags)
    torch.cuda.synchronize()
    for t in range(steps):
        for i, (K, N) in enumerate(shapes):
            packed, alpha, codes, a_ref = quant[i]
            _, _, _, y_r = oracle.forward(xo_all[t][i], codes, a_ref)
            assert_y_close(np_(ys[t][i]), y_r)


# ---------------------------------------------------------------- failure detection
def test_bounded_wait_reports_timeout():
    """A wait on an mbarrier that nothing completes gives up after its bound,
    records BL_ERR_TIMEOUT in the device error word and returns; the context
    stays usable."""
    import bitlinear_w1_a8_03_b200 as bl
    assert bl.bitlinear_device_error() == 0
    bl.check(bl.lib().bitlinear_selftest_timeout(2000, torch.cuda.current_stream().cuda_stream), "selftest")
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 9
    assert bl.bitlinear_device_error() == 0  # read clears it
    t = torch.ones(1000, device="cuda")
    assert float(t.sum()) == 1000.0


def test_linear_right_after_weight_quantisation_without_sync():
    """Default flags: the product kernel may not read weights that work still
    in flight is writing, so quantising and using them back to back with no
    host synchronisation must give the oracle's result."""
    import bitlinear_w1_a8_03_b200 as bl
    K, N = 4096, 2048
    W = synth.weights(31, N, K, 0.02)
    x = synth.activations(31, 1, K, outliers=True)
    Wd, Wo = as_input(W, "f32")
    xd, xo = as_input(x, "bf16")
    torch.cuda.synchronize()
    for rep in range(3):
        packed = torch.empty((N, bl.packed_row_bytes(K)), dtype=torch.uint8, device="cuda")
        packed.fill_(0xAA)  # garbage a premature read would see
        alpha = torch.empty(1, dtype=torch.float32, device="cuda")
        bl.bitlinear_quantize_weights(Wd, W_packed=packed, alpha=alpha)
        y = bl.bitlinear_linear(xd, packed, alpha, N)
        _, a_ref, codes = oracle.quantize_weights(Wo)
        _, _, _, y_r = oracle.forward(xo, codes, a_ref)
        assert_y_close(np_(y), y_r)


def _near_half_integer_rows(beta_target, rows, K, seed):
    """Rows whose max |x| is beta_target and whose other values put 127·x/β
    next to a half-integer k + 1/2 (the rounding boundaries): a few ulps away,
    just outside and inside a 1e-4 band, or anywhere."""
    rng = np.random.default_rng(seed)
    x = np.empty((rows, K), dtype=np.float32)
    for r in range(rows):
        k = rng.integers(-127, 127, size=K).astype(np.float64)
        kind = rng.integers(0, 4, size=K)
        off = np.choose(kind, [np.zeros(K), rng.choice([-1.1e-4, 1.1e-4, -0.9e-4, 0.9e-4], size=K),
                               rng.uniform(-3e-4, 3e-4, size=K), rng.uniform(-0.5, 0.5, size=K)])
        v = ((k + 0.5 + off) * beta_target / 127.0).astype(np.float32)
        steps = np.where(kind == 0, rng.integers(-3, 4, size=K), 0)
        for s in range(1, 4):
            v = np.where(steps >= s, np.nextafter(v, np.float32(np.inf)), v)
            v = np.where(steps <= -s, np.nextafter(v, np.float32(-np.inf)), v)
        v[rng.integers(0, K)] = np.float32(beta_target) * (1 if r % 2 else -1)
        x[r] = np.clip(v, -beta_target, beta_target)
    return x


@pytest.mark.parametrize("rows", [3, 400])
@pytest.mark.parametrize("beta_target", [3.0, 0.7, 1e-3, 12345.678, 127.0])
def test_act_quant_rounding_boundaries(rows, beta_target):
    """Quotients 127·x/β next to k + 1/2 decide the int8 code: bit-exact with
    the oracle's correctly rounded division, in few-row and many-row launches."""
    x = _near_half_integer_rows(beta_target, rows, 1024, seed=int(beta_target * 1000) + rows)
    for dtype in ("f32", "bf16"):
        xd, xo = as_input(x, dtype)
        xq, beta = bl.bitlinear_quantize_act(xd)
        xq_r, beta_r = oracle.quantize_act(xo)
        assert np.array_equal(np_(beta), beta_r)
        assert np.array_equal(np_(xq), xq_r)


def _grouped_linear_case(shapes, M, dtype, seed, flags=0):
    """Grouped linear over `shapes` [(K, N)] at M tokens: x̃, β, acc and y of
    every problem bit-exact against the oracle."""
    probs, refs = [], []
    for i, (K, N) in enumerate(shapes):
        W = synth.weights(seed + 17 * i, N, K, 0.02)
        x = synth.activations(seed + 17 * i + 1, M, K, outliers=True)
        packed, alpha, codes, a_ref = check_weights(W, "f32")
        xd, xo = as_input(x, dtype)
        pr = dict(x=xd, x_q=torch.empty((M, K), dtype=torch.int8, device="cuda"),
                  beta=torch.empty(M, dtype=torch.float32, device="cuda"), W_packed=packed, alpha=alpha, N=N,
                  y=torch.empty((M, N), dtype=torch.float32, device="cuda"),
                  acc_out=torch.empty((M, N), dtype=torch.int32, device="cuda"))
        probs.append(pr)
        refs.append(oracle.forward(xo, codes, a_ref))
    bl.bitlinear_linear_grouped(probs, flags=flags)
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    for pr, (xq_r, beta_r, acc_r, y_r) in zip(probs, refs):
        assert np.array_equal(np_(pr["x_q"]), xq_r)
        assert np.array_equal(np_(pr["beta"]), beta_r)
        assert np.array_equal(np_(pr["acc_out"]), acc_r)
        assert_y_close(np_(pr["y"]), y_r)


@pytest.mark.parametrize("M", [1, 2, 4])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fused_linear_grouped(M, dtype, fusion):
    """Few tokens: the product kernel quantises x itself (one launch) when
    fused; the same results either way."""
    # 11008-wide float32 rows take the prologue's two-pass branch
    _grouped_linear_case([(4096, 300), (1024, 700), (4096 + 64, 129), (11008, 200)], M, dtype, seed=9100 + M)


def test_linear_grouped_many_small_problems(fusion):
    """Sixteen tiny problems: some CTA ranges meet more than two problems, so
    even forced fusion falls back to the separate quantisation kernel."""
    _grouped_linear_case([(256 + 64 * (i % 3), 24 + 8 * i) for i in range(16)], 1, "bf16", seed=9200)


def test_linear_rows_wider_than_a_fused_slot(fusion):
    """Two tokens of a 28672-wide row exceed the fused slot: separate kernels."""
    _grouped_linear_case([(28672, 96)], 2, "bf16", seed=9300, flags=1)


@pytest.mark.parametrize("M", [1, 3])
def test_linear_block_fused_and_not(M, fusion):
    """bitlinear_linear_block with shared and summed inputs (x = a + b), the
    stack's first call shape, against the oracle."""
    K, N = 1024, [512, 256, 768]
    a = synth.activations(9400 + M, M, K, outliers=True)
    b = synth.activations(9500 + M, M, K, outliers=False)
    x = (a + b).astype(np.float32)
    xs = torch.empty((M, K), dtype=torch.float32, device="cuda")
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    beta = torch.empty(M, dtype=torch.float32, device="cuda")
    fwds, refs = [], []
    for i, n in enumerate(N):
        W = synth.weights(9600 + i, n, K, 0.02)
        packed, alpha, codes, a_ref = check_weights(W, "f32")
        fwds.append(dict(x_q=xq, beta=beta, W_packed=packed, alpha=alpha, N=n,
                         y=torch.empty((M, n), dtype=torch.float32, device="cuda")))
        refs.append(oracle.forward(x, codes, a_ref))
    bl.bitlinear_linear_block([dict(a=dev_f32(a), b=dev_f32(b), x_sum=xs, x_q=xq, beta=beta)], fwds,
                              flags=bl.BL_LINEAR_WEIGHTS_STATIC)
    torch.cuda.synchronize()
    assert bl.bitlinear_device_error() == 0
    assert np.array_equal(np_(xs), x)
    assert np.array_equal(np_(xq), refs[0][0]) and np.array_equal(np_(beta), refs[0][1])
    for f, (_, _, _, y_r) in zip(fwds, refs):
        assert_y_close(np_(f["y"]), y_r)
