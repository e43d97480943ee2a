"""Launch order: inputs written by the kernel just before a call, buffers reused call after call.

The scale transform, the scale-layout pass and the GEMM are launched with programmatic stream
serialisation, so each may start while the kernel before it still runs (the quantiser is not,
but the layout pass after it is).
Each waits for that kernel before it reads what that kernel may write or writes what it may
read; the GEMM reads its operands (and the grouped kernels their expert indices or counts)
before it waits, which is sound only because the layout pass lets it start once every kernel
ahead has completed.  These tests put that to work: on a side stream, behind a long kernel,
ordinary torch kernels write the operands, scales, indices, counts or the quantiser's input
immediately before each call, two input sets alternate, the library's packed-scale buffers (or
the fixed scratch of the no-allocation entry point) are reused by the next call, and a torch
kernel copies D right after.  Every result must equal, bit for bit, the one computed for its
input set with synchronisations around the call, and that one is checked against the fp64
oracle first.
"""

import ctypes

import numpy as np
import pytest

import inputs

from parity import bf16_to_f64, check_gemm, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ROUNDS = 24
SENTINEL = 0x3C5A  # bf16 bits left in masked rows that are not written


@pytest.fixture(scope="module")
def ops():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import block_scaled_precision_sm_b200.ops as ops

    assert ops.device_status() == 0
    return ops


@pytest.fixture(scope="module")
def busy():
    # 256 MB: one pass over it keeps the stream busy for ~100 us, so the kernels queued behind
    # it are launched early and wait
    return torch.zeros(1 << 26, dtype=torch.float32, device="cuda")


def _same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


def _run_rounds(busy, prepare, call, n_sets):
    """On a side stream: long kernel, `prepare(i)` (torch writes of set i % n_sets), `call(i)` ->
    D, then a copy of D; returns the copies once the stream has drained."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    outs = []
    with torch.cuda.stream(side):
        for i in range(ROUNDS):
            busy.add_(1.0)
            prepare(i % n_sets)
            outs.append(call(i % n_sets).clone())
    torch.cuda.synchronize()
    return outs


# dense FP8: transposed K halves on a cluster (M = 128), CTA-pair tiles, and a split last wave
# whose counters the layout pass zeroes
@pytest.mark.parametrize("m,n,k", [(128, 1024, 2048), (384, 672, 1024), (256, 7168, 2048)])
def test_dense_inputs_written_just_before_each_call(ops, orc, busy, m, n, k):
    probs = [inputs.dense_fp8_problem(m, n, k, seed=s) for s in (31, 32)]
    B = to_dev(probs[0]["B"])  # one weight, two activation and scale sets
    src = [{key: to_dev(p[key]) for key in ("A", "sfa", "sfb")} for p in probs]
    refs = []
    for p, s in zip(probs, src):
        torch.cuda.synchronize()
        D = ops.gemm_fp8_nt(s["A"], s["sfa"], B, s["sfb"])
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        check_gemm(bf16_to_f64(D), orc.gemm_fp8(p["A"], p["sfa"], probs[0]["B"], p["sfb"]), f"{m}x{n}x{k}")
        refs.append(D)
    A_buf = torch.empty_like(src[0]["A"])
    sfa_buf, sfb_buf = torch.empty_like(src[0]["sfa"]), torch.empty_like(src[0]["sfb"])
    D_buf = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")

    def prepare(j):
        A_buf.copy_(src[j]["A"])
        sfa_buf.copy_(src[j]["sfa"])
        sfb_buf.copy_(src[j]["sfb"])

    # uint8 scales: transform, transform, layout pass, GEMM, each packed buffer reused next call
    outs = _run_rounds(busy, prepare, lambda j: ops.gemm_fp8_nt(A_buf, sfa_buf, B, sfb_buf, D_buf), 2)
    assert ops.device_status() == 0
    for i, D in enumerate(outs):
        assert _same_bits(D, refs[i % 2]), f"uint8 scales, round {i}"

    # packed scales: the copy of A is the kernel right before the layout pass
    packed = [(ops.transform_sf_ue8m0(s["sfa"]), ops.transform_sf_ue8m0(s["sfb"])) for s in src]
    outs = _run_rounds(busy, lambda j: A_buf.copy_(src[j]["A"]),
                       lambda j: ops.gemm_fp8_nt(A_buf, packed[j][0], B, packed[j][1], D_buf), 2)
    assert ops.device_status() == 0
    for i, D in enumerate(outs):
        assert _same_bits(D, refs[i % 2]), f"packed scales, round {i}"


def test_no_alloc_scratch_reused_by_the_next_call(ops, orc, busy):
    from block_scaled_precision_sm_b200 import _lib

    lib = _lib.load()
    m, n, k = 96, 1000, 1024
    probs = [inputs.dense_fp8_problem(m, n, k, seed=s, b_block_rows=1) for s in (41, 42)]
    B = to_dev(probs[0]["B"])
    src = [{key: to_dev(p[key]) for key in ("A", "sfa", "sfb")} for p in probs]
    A_buf = torch.empty_like(src[0]["A"])
    sfa_buf, sfb_buf = torch.empty_like(src[0]["sfa"]), torch.empty_like(src[0]["sfb"])
    D_buf = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    vp = lambda t: ctypes.c_void_p(t.data_ptr())

    def call(_):
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        rc = lib.gemm_fp8_nt_noalloc(vp(A_buf), vp(sfa_buf), vp(B), vp(sfb_buf), vp(D_buf), vp(status), m, n, k,
                                     A_buf.stride(0), B.stride(0), D_buf.stride(0), sfa_buf.stride(0),
                                     sfb_buf.stride(0), 1, stream)
        assert rc == 0
        return D_buf

    def prepare(j):
        A_buf.copy_(src[j]["A"])
        sfa_buf.copy_(src[j]["sfa"])
        sfb_buf.copy_(src[j]["sfb"])

    refs = []
    for j, p in enumerate(probs):
        torch.cuda.synchronize()
        prepare(j)
        D = call(j).clone()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        check_gemm(bf16_to_f64(D), orc.gemm_fp8(p["A"], p["sfa"], probs[0]["B"], p["sfb"], gran_n=1), "no-alloc")
        refs.append(D)
    outs = _run_rounds(busy, prepare, call, 2)
    assert int(status.item()) == 0
    for i, D in enumerate(outs):
        assert _same_bits(D, refs[i % 2]), f"no-alloc, round {i}"


def test_grouped_indices_written_just_before_each_call(ops, orc, busy):
    # two routings with the same padded row count: 128 + 0 + 256 + 128 and 128 + 256 + 128 + 0
    n, k = 448, 512
    probs = [inputs.grouped_fp8_problem(4, 0, n, k, seed=s, counts=c)
             for s, c in ((51, [100, 0, 150, 50]), (52, [128, 200, 60, 0]))]
    assert probs[0]["M"] == probs[1]["M"] == 512
    B, sfb = to_dev(probs[0]["B"]), to_dev(probs[0]["sfb"])
    src = [{key: to_dev(p[key]) for key in ("A", "sfa", "m_indices")} for p in probs]
    refs = []
    for p, s in zip(probs, src):
        torch.cuda.synchronize()
        D = ops.m_grouped_gemm_fp8_nt_contiguous(s["A"], s["sfa"], B, sfb, s["m_indices"])
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        valid = p["m_indices"] >= 0
        ref = orc.gemm_grouped_fp8(p["A"], p["sfa"], probs[0]["B"], probs[0]["sfb"], p["m_indices"])
        check_gemm(bf16_to_f64(D)[valid], ref[valid], "grouped")
        refs.append(D)
    A_buf, sfa_buf, idx_buf = (torch.empty_like(src[0][key]) for key in ("A", "sfa", "m_indices"))
    D_buf = torch.empty((512, n), dtype=torch.bfloat16, device="cuda")

    def prepare(j):
        A_buf.copy_(src[j]["A"])
        sfa_buf.copy_(src[j]["sfa"])
        idx_buf.copy_(src[j]["m_indices"])

    outs = _run_rounds(busy, prepare,
                       lambda j: ops.m_grouped_gemm_fp8_nt_contiguous(A_buf, sfa_buf, B, sfb, idx_buf, D_buf), 2)
    assert ops.device_status() == 0
    for i, D in enumerate(outs):
        assert _same_bits(D, refs[i % 2]), f"grouped, round {i}"


def test_masked_counts_written_just_before_each_call(ops, orc, busy):
    n, k, max_m = 704, 512, 384
    p = inputs.masked_fp8_problem(3, max_m, n, k, seed=61, counts=[300, 17, 0])
    A, sfa, B, sfb = (to_dev(p[key]) for key in ("A", "sfa", "B", "sfb"))
    counts = [to_dev(np.array(c, np.int32)) for c in ([300, 17, 0], [5, 384, 129])]
    refs = []
    for c in counts:
        torch.cuda.synchronize()
        D = torch.full((3, max_m, n), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        ops.m_grouped_gemm_fp8_nt_masked(A, sfa, B, sfb, c, D)
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        c_h = c.cpu().numpy()
        valid = np.concatenate([np.arange(max_m) < x for x in c_h])
        raw = D.view(torch.int16).cpu().numpy().view(np.uint16).reshape(3 * max_m, n)
        assert (raw[~valid] == SENTINEL).all()
        ref = orc.gemm_masked_fp8(p["A"], p["sfa"], p["B"], p["sfb"], c_h)
        check_gemm(bf16_to_f64(D).reshape(3 * max_m, n)[valid], ref[valid], f"masked {c_h.tolist()}")
        refs.append(D)
    cnt_buf = torch.empty_like(counts[0])
    D_buf = torch.empty((3, max_m, n), dtype=torch.bfloat16, device="cuda")

    def prepare(j):
        D_buf.view(torch.int16).fill_(SENTINEL)
        cnt_buf.copy_(counts[j])

    outs = _run_rounds(busy, prepare, lambda j: ops.m_grouped_gemm_fp8_nt_masked(A, sfa, B, sfb, cnt_buf, D_buf), 2)
    assert ops.device_status() == 0
    for i, D in enumerate(outs):
        assert _same_bits(D, refs[i % 2]), f"masked, round {i}"


@pytest.mark.parametrize("m,n,k", [(128, 1024, 2048), (384, 672, 1024)])
def test_quantiser_output_read_by_the_next_call(ops, orc, busy, m, n, k):
    # quantise (fp32 activations, 1 x 128 blocks) and multiply, with nothing between the two calls
    pb = inputs.dense_fp8_problem(m, n, k, seed=71)
    B, sfb = to_dev(pb["B"]), ops.transform_sf_ue8m0(to_dev(pb["sfb"]))
    xs = [inputs.normal_matrix(m, k, seed=s) for s in (72, 73)]
    src = [to_dev(x) for x in xs]
    refs = []
    for x, xd in zip(xs, src):
        torch.cuda.synchronize()
        q, sf = ops.quantize_fp8(xd)
        D = ops.gemm_fp8_nt(q, sf, B, sfb)
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        qa, ea = orc.quantize_fp8(x, 1)
        check_gemm(bf16_to_f64(D), orc.gemm_fp8(qa, ea, pb["B"], pb["sfb"]), f"quantise + gemm {m}x{n}x{k}")
        refs.append(D)
    x_buf = torch.empty_like(src[0])
    q_buf = torch.empty((m, k), dtype=torch.uint8, device="cuda")
    sf_buf = torch.empty(((k // 128 + 1) // 2, ops.sf_ld(m)), dtype=torch.int16, device="cuda")
    D_buf = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")

    def call(j):
        ops.quantize_fp8(x_buf, q=q_buf, sf=sf_buf)
        return ops.gemm_fp8_nt(q_buf, sf_buf, B, sfb, D_buf)

    outs = _run_rounds(busy, lambda j: x_buf.copy_(src[j]), call, 2)
    assert ops.device_status() == 0
    for i, D in enumerate(outs):
        assert _same_bits(D, refs[i % 2]), f"quantise + gemm, round {i}"
