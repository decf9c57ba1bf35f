"""The C ABI without a GPU: exports, status strings, planning, and the
argument checks that must reject a call before anything is launched."""
import ctypes

import pytest


def test_library_exports_every_declared_entry_point(fk):
    names = fk.header_functions()
    assert set(names) >= {"fk_gelu_tanh", "fk_softmax_rows", "fk_softmax_rows_ex",
                          "fk_softmax_rows_plan", "fk_status_string", "fk_last_cuda_error",
                          "fk_version", "fk_wait_timeouts", "fk_wait_selftest",
                          "fk_softmax_rows_workspace", "fk_softmax_rows_ws"}
    lib = ctypes.CDLL(fk.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(fk):
    assert fk.fk_version() == 10000
    for code, word in [(0, "FK_OK"), (1, "INVALID_ARG"), (2, "DTYPE"), (3, "DEVICE"), (4, "CUDA")]:
        assert word in fk.fk_status_string(code)
    assert "unknown" in fk.fk_status_string(99)


@pytest.mark.parametrize("rows,cols,dtype,expect", [
    (256, 1000, 0, ("warp", 64, 8, 1)),         # 256x1000 fp32: two rows per block
    (8192, 4096, 0, ("cta", 128, 8, 1)),        # 8192x4096 fp32
    (1 << 20, 2048, 1, ("cta", 128, 2, 1)),     # bf16 attention rows
    (512, 131072, 0, ("cluster", 128, 16, 16)), # vocab-sized rows
    (4, 1, 0, ("warp", 64, 1, 1)),
    (4, 128, 0, ("warp", 64, 1, 1)),
    (4, 129, 0, ("warp", 64, 2, 1)),
    (4, 1024, 0, ("warp", 64, 8, 1)),
    (588, 1000, 0, ("warp", 64, 8, 1)),         # 147 blocks of 4 rows leave an SM idle
    (589, 1000, 0, ("warp", 128, 8, 1)),
    (1176, 1000, 0, ("warp", 128, 8, 1)),
    (1177, 1000, 0, ("warp", 256, 8, 1)),       # 148 blocks of 8 rows
    (4, 1025, 0, ("cta", 128, 8, 1)),
    (4, 2049, 1, ("cta", 128, 4, 1)),        # bf16 past 2048 columns: 32 values a thread
    (4, 8192, 0, ("cta", 256, 8, 1)),
    (4, 8193, 0, ("cluster", 128, 16, 2)),     # wider rows: clusters of 128-thread blocks
    (4, 8192, 1, ("cta", 256, 4, 1)),
    (4, 8193, 1, ("cluster", 128, 8, 2)),
    (4, 1024, 1, ("warp", 64, 4, 1)),
    (4, 16385, 1, ("cluster", 128, 8, 3)),
    (4, 32768, 0, ("cluster", 128, 16, 4)),
    (4, 32769, 0, ("cluster", 128, 16, 5)),
    (4, 131073, 0, ("cluster", 256, 16, 9)),
    (4, 524288, 0, ("cluster", 512, 16, 16)),
    (3, 524289, 0, ("split", 512, 4, 1)),
    (4, 524289, 0, ("twophase", 512, 4, 16)),
    (64, 524289, 0, ("twophase", 512, 4, 16)),
    (64, 1 << 22, 0, ("split", 512, 4, 1)),
    (2, 524289, 1, ("split", 512, 2, 1)),
    (100, 524289, 1, ("twophase", 512, 2, 16)),
    (4, 524288, 1, ("cluster", 512, 8, 16)),
])
def test_auto_plans(fk, rows, cols, dtype, expect):
    p = fk.fk_softmax_rows_plan(rows, cols, dtype).as_dict()
    assert (p["path"], p["threads"], p["vpt"], p["cluster"]) == expect


def test_warp_rows_per_block_follow_the_rule(fk):
    """The warp path's rows per block (threads / 32): the largest of 8, 4, 2
    whose grid still gives each of the B200's 148 SMs a block, 2 at the
    least, for every row count and both dtypes (LayerNorm takes the same)."""
    for dtype in (0, 1):
        for rows in list(range(1, 1300, 7)) + [1183, 1184, 1185, 4096, 1 << 20]:
            t = fk.fk_softmax_rows_plan(rows, 1000, dtype).as_dict()["threads"]
            want = 8
            while want > 2 and -(-rows // want) < 148:
                want //= 2
            assert t == 32 * want, (dtype, rows, t)
            assert fk.fk_layernorm_rows_plan(rows, 1000, dtype).as_dict()["threads"] == t


def _softmax_rule(rows, cols, dtype):
    """The documented automatic softmax plan, restated: a warp per row up to
    1024 columns; one block per row up to 8192 (bf16 rows of up to 2048
    columns 16 values a thread, every other row 32; the fewest threads from
    128 that hold the row); clusters of blocks with 64 values a thread up to
    524288 (the smallest block from 128 threads whose cluster of at most 16
    holds the row, at least 2 blocks); past that the split path for fewer
    than 4 rows or 4M columns and more, else the two-phase path."""
    vec = 4 if dtype == 0 else 8
    if cols <= 1024:
        vpt = 1
        while 32 * vpt * vec < cols:
            vpt *= 2
        return ("warp", vpt, 1)
    if cols <= 8192:
        ept = 16 if dtype == 1 and cols <= 2048 else 32
        t = 128
        while t * ept < cols:
            t *= 2
        return ("cta", t, ept // vec, 1)
    if cols <= 16 * 512 * 64:
        t = 128
        k = -(-cols // (t * 64))
        while k > 16:
            t *= 2
            k = -(-cols // (t * 64))
        return ("cluster", t, 64 // vec, max(k, 2))
    return ("split",) if rows < 4 or cols >= 1 << 22 else ("twophase",)


def test_softmax_auto_plans_follow_the_rule(fk):
    widths = sorted({1, 7, 64, 100, 128, 129, 513, 1000, 1024, 1025, 2047, 2048, 2049, 4095, 4096, 4097,
                     8191, 8192, 8193, 16384, 16385, 32768, 32769, 65536, 131072, 131073, 262144, 262145,
                     524288, 524289, 1 << 21, (1 << 22) - 1, 1 << 22})
    for dtype in (0, 1):
        for rows in (1, 3, 4, 5000):
            for cols in widths:
                p = fk.fk_softmax_rows_plan(rows, cols, dtype).as_dict()
                want = _softmax_rule(rows, cols, dtype)
                got = (p["path"],) + ((p["vpt"], p["cluster"]) if p["path"] == "warp" else
                                       (p["threads"], p["vpt"], p["cluster"]) if p["path"] in ("cta", "cluster")
                                       else ())
                assert got == want, (rows, cols, dtype, p, want)
                # whatever the path, a row is held (or streamed) whole
                if p["path"] in ("cta", "cluster"):
                    assert p["threads"] * p["vpt"] * (4 if dtype == 0 else 8) * p["cluster"] >= cols


def test_forced_plans_and_capacity_errors(fk):
    P = fk
    assert P.fk_softmax_rows_plan(2, 100, 0, P.FK_PATH_TWOPHASE).as_dict()["cluster"] == 1
    assert P.fk_softmax_rows_plan(2, 100, 0, P.FK_PATH_CLUSTER).as_dict()["cluster"] == 2
    assert P.fk_softmax_rows_plan(2, 100, 0, P.FK_PATH_CTA).as_dict()["threads"] == 128
    with pytest.raises(P.FkError):
        P.fk_softmax_rows_plan(2, 1025, 0, P.FK_PATH_WARP)
    with pytest.raises(P.FkError):
        P.fk_softmax_rows_plan(2, 32769, 0, P.FK_PATH_CTA)
    with pytest.raises(P.FkError):
        P.fk_softmax_rows_plan(2, 16 * 32768 + 1, 0, P.FK_PATH_CLUSTER)
    with pytest.raises(P.FkError) as e:
        P.fk_softmax_rows_plan(2, 10, 7)
    assert e.value.status == P.FK_ERR_UNSUPPORTED_DTYPE
    with pytest.raises(P.FkError):
        P.fk_softmax_rows_plan(2, 0, 0)


# Fake addresses: never dereferenced.  Without a GPU the checks end at
# "no device"; on a GPU machine the pointer-attribute query rejects them.
A, B = 0x10000000, 0x20000000
REJECT_NO_LAUNCH = {1, 3}


def test_zero_sizes_are_noops_even_with_null(fk):
    assert fk.fk_gelu_tanh(0, 0, 0, 0) == fk.FK_OK
    assert fk.fk_softmax_rows(0, 0, 0, 10, 0, 0) == fk.FK_OK
    assert fk.fk_softmax_rows(0, 0, 10, 0, 1, 0) == fk.FK_OK


def test_null_pointers_with_nonzero_size(fk):
    assert fk.fk_gelu_tanh(0, B, 10, 0) == fk.FK_ERR_INVALID_ARG
    assert fk.fk_gelu_tanh(A, 0, 10, 0) == fk.FK_ERR_INVALID_ARG
    assert fk.fk_softmax_rows(0, B, 4, 4, 0, 0) == fk.FK_ERR_INVALID_ARG


def test_bad_dtype_is_reported_first(fk):
    assert fk.fk_softmax_rows(A, B, 4, 4, 2, 0) == fk.FK_ERR_UNSUPPORTED_DTYPE
    assert fk.fk_softmax_rows(A, B, 0, 4, -1, 0) == fk.FK_ERR_UNSUPPORTED_DTYPE


def test_misaligned_and_overflowing_and_overlapping_arguments(fk):
    assert fk.fk_gelu_tanh(A + 1, B, 10, 0) == fk.FK_ERR_INVALID_ARG          # not 4-byte aligned
    assert fk.fk_softmax_rows(A, B + 1, 4, 4, 1, 0) == fk.FK_ERR_INVALID_ARG  # bf16, odd address
    assert fk.fk_softmax_rows(A, B, 1 << 62, 1 << 3, 0, 0) == fk.FK_ERR_INVALID_ARG  # bytes overflow
    assert fk.fk_gelu_tanh(A, A + 4, 16, 0) == fk.FK_ERR_INVALID_ARG         # partial overlap
    assert fk.fk_softmax_rows(A, A + 64, 4, 32, 0, 0) == fk.FK_ERR_INVALID_ARG


def test_valid_looking_arguments_without_a_usable_device_are_rejected(fk):
    assert fk.fk_gelu_tanh(A, B, 10, 0) in REJECT_NO_LAUNCH
    assert fk.fk_gelu_tanh(A, A, 10, 0) in REJECT_NO_LAUNCH                   # in place
    assert fk.fk_softmax_rows(A, B, 4, 4, 0, 0) in REJECT_NO_LAUNCH


def test_explicit_plan_validation(fk):
    bad = [fk.make_plan(fk.FK_PATH_WARP, threads=96),
           fk.make_plan(fk.FK_PATH_WARP, threads=512),
           fk.make_plan(fk.FK_PATH_WARP, vpt=3),
           fk.make_plan(fk.FK_PATH_CTA, threads=96),
           fk.make_plan(fk.FK_PATH_CLUSTER, cluster=17),
           fk.make_plan(fk.FK_PATH_CLUSTER, cluster=1),
           fk.make_plan(fk.FK_PATH_TWOPHASE, threads=256),
           fk.make_plan(9)]
    for p in bad:
        assert fk.fk_softmax_rows_ex(A, B, 4, 64, 0, p, 0) == fk.FK_ERR_INVALID_ARG, p
    # a plan that cannot hold the row
    assert fk.fk_softmax_rows_ex(A, B, 4, 5000, 0, fk.make_plan(fk.FK_PATH_CTA, threads=128), 0) \
        == fk.FK_ERR_INVALID_ARG


def test_wait_entry_points_check_arguments_first(fk):
    assert fk.lib().fk_wait_selftest(0, None) == fk.FK_ERR_INVALID_ARG
    assert fk.lib().fk_wait_selftest(10_000_001, None) == fk.FK_ERR_INVALID_ARG
    assert fk.lib().fk_wait_timeouts(None, 0) == fk.FK_ERR_INVALID_ARG


def test_cluster_plan_validation(fk):
    P = fk
    # 64 values per thread fit blocks of at most 512 threads
    ok = P.make_plan(P.FK_PATH_CLUSTER, threads=512, vpt=16, cluster=16)
    bad = P.make_plan(P.FK_PATH_CLUSTER, threads=1024, vpt=16, cluster=16)
    assert P.fk_softmax_rows_ex(A, B, 4, 1000, 0, bad, 0) == P.FK_ERR_INVALID_ARG
    assert P.fk_softmax_rows_ex(A, B, 4, 1000, 0, ok, 0) in REJECT_NO_LAUNCH


def test_split_plan_and_workspace(fk):
    P = fk
    p = P.fk_softmax_rows_plan(1, 64 << 20, P.FK_F32).as_dict()
    assert p["path"] == "split" and p["chunks"] >= 148
    # the workspace holds one (max, sum) pair per chunk of the rows of a launch
    ws = P.fk_softmax_rows_workspace(1, 64 << 20, P.FK_F32)
    assert ws == 8 * p["chunks"]
    assert P.fk_softmax_rows_workspace(8192, 4096, P.FK_F32) == 0
    assert P.fk_softmax_rows_workspace(512, 131072, P.FK_BF16) == 0
    big = P.fk_softmax_rows_workspace(10 ** 6, 1 << 20, P.FK_F32, P.make_plan(P.FK_PATH_SPLIT))
    assert 0 < big <= 8 << 20
    # forced split for a short row: one chunk
    q = P.fk_softmax_rows_plan(3, 100, P.FK_BF16, P.FK_PATH_SPLIT).as_dict()
    assert q["path"] == "split" and q["chunks"] == 1
    # explicit chunk counts other than the derived one are refused
    assert P.fk_softmax_rows_ex(A, B, 3, 100, 0, P.make_plan(P.FK_PATH_SPLIT, chunks=7), 0) \
        == P.FK_ERR_INVALID_ARG
    # a caller workspace that is too small is refused before anything else runs
    assert P.fk_softmax_rows_ws(A, B, 1, 1 << 22, 0, None, 0x30000000, 8, 0) == P.FK_ERR_INVALID_ARG or \
        P.fk_softmax_rows_ws(A, B, 1, 1 << 22, 0, None, 0x30000000, 8, 0) in REJECT_NO_LAUNCH
    with pytest.raises(P.FkError):
        P.fk_softmax_rows_workspace(1, 10, 9)


NOALLOC_PAIRS = 131072  # the allocation-free entry point's scratch: 1 MiB of (max, sum) pairs


@pytest.mark.parametrize("dtype", [0, 1])
def test_noalloc_batches_fit_its_scratch_array(fk, dtype):
    """fk_softmax_rows_noalloc runs split-path shapes in batches of
    floor(131072 / chunks) rows, each batch planned for its own row count.
    Every batch size it can form -- the full batch and every shorter last
    batch -- must need at most the array's 1 MiB of workspace (host-only
    planning through the C ABI).  The multi-batch loop engages only when
    rows * chunks exceeds 131072, e.g. more than 8192 rows of 4M columns
    (64 GiB of bf16 input), so this planning check is how it is tested."""
    P = fk
    split = P.make_plan(P.FK_PATH_SPLIT)
    for cols in (524289, 1 << 20, 3_000_001, 1 << 22, 5_000_001, 1 << 24, 1 << 28, 1 << 35):
        for rows in (1, 2, 3, 4, 7, 64, 1183, 1184, 1185, 5000, 8192, 8193, 20000, 100_000, 1_000_003):
            plan = P.fk_softmax_rows_plan(rows, cols, dtype).as_dict()
            if plan["path"] != "split":
                continue
            per_batch = NOALLOC_PAIRS // plan["chunks"]
            assert per_batch >= 1
            last = rows % per_batch
            sizes = {min(per_batch, rows), last or per_batch, 1}
            sizes |= {n for n in (2, 3, 4, 100, 1183, 1184, 1185) if n <= min(per_batch, rows)}
            for n in sizes:
                need = P.fk_softmax_rows_workspace(n, cols, dtype, split)
                assert 0 < need <= NOALLOC_PAIRS * 8, (rows, cols, n, need)
    # the longest row the array serves: 2^35 elements in 131072 chunks
    assert P.fk_softmax_rows_plan(1, 1 << 35, dtype, P.FK_PATH_SPLIT).as_dict()["chunks"] == NOALLOC_PAIRS
    assert P.fk_softmax_rows_plan(1, (1 << 35) + 1, dtype, P.FK_PATH_SPLIT).as_dict()["chunks"] > NOALLOC_PAIRS


@pytest.mark.parametrize("dtype", [0, 1])
def test_noalloc_capacity_is_checked_before_the_device(fk, dtype):
    """fk_softmax_rows_noalloc_cap refuses a capacity outside 1 .. 131072,
    or one that cannot hold a batch as it is planned, before it looks at the
    pointers or the device (so null pointers are enough here)."""
    P = fk
    rows, cols = 80, 1 << 22
    assert P.fk_softmax_rows_noalloc_cap(0, 0, rows, cols, dtype, 0, 0) == P.FK_ERR_INVALID_ARG
    assert P.fk_softmax_rows_noalloc_cap(0, 0, rows, cols, dtype, NOALLOC_PAIRS + 1, 0) == P.FK_ERR_INVALID_ARG
    chunks = P.fk_softmax_rows_plan(rows, cols, dtype).as_dict()["chunks"]
    assert P.fk_softmax_rows_noalloc_cap(0, 0, rows, cols, dtype, chunks - 1, 0) == P.FK_ERR_INVALID_ARG
    # a capacity that holds the batch size as planned for all rows, but not
    # the batch as its own row count plans it (fewer rows, more chunks each)
    split = P.make_plan(P.FK_PATH_SPLIT)
    rows2, cap = 112, 592
    per = cap // P.fk_softmax_rows_plan(rows2, cols, dtype).as_dict()["chunks"]
    assert per >= 1 and P.fk_softmax_rows_workspace(per, cols, dtype, split) > cap * 8
    assert P.fk_softmax_rows_noalloc_cap(0, 0, rows2, cols, dtype, cap, 0) == P.FK_ERR_INVALID_ARG
    assert P.fk_softmax_rows_noalloc_cap(0, 0, rows, cols, 9, 1200, 0) == P.FK_ERR_UNSUPPORTED_DTYPE
    assert P.fk_softmax_rows_noalloc_cap(0, 0, 0, cols, dtype, 1200, 0) == P.FK_OK  # empty: no-op


def _layernorm_rule(cols, dtype):
    """The documented LayerNorm plan: one warp per row up to 1024 columns;
    one block per row up to 32768 (16 values per thread up to 2048 columns,
    else 32; the fewest threads from 128 up that hold the row); a 512-thread
    streaming block above.  vpt counts 16-byte vectors (4 fp32 or 8 bf16)."""
    vec = 4 if dtype == 0 else 8
    if cols <= 1024:
        return "warp"
    if cols <= 32768:
        ept = 16 if cols <= 128 * 16 else 32
        threads = 128
        while threads * ept < cols:
            threads *= 2
        return ("cta", threads, ept // vec)
    return ("twophase", 512, 16 // vec)


@pytest.mark.parametrize("cols", [1, 1024, 1025, 2048, 2049, 4096, 4097, 8193, 16384, 16385, 32768, 32769, 1 << 20])
@pytest.mark.parametrize("dtype", [0, 1])
def test_layernorm_auto_plans_follow_the_rule(fk, cols, dtype):
    p = fk.fk_layernorm_rows_plan(64, cols, dtype).as_dict()
    want = _layernorm_rule(cols, dtype)
    if want == "warp":
        vec = 4 if dtype == 0 else 8
        assert p["path"] == "warp" and p["cluster"] == 1
        assert p["vpt"] * vec * 32 >= cols  # the warp's 32 lanes hold the row
    else:
        assert (p["path"], p["threads"], p["vpt"]) == want and p["cluster"] == 1


def test_layernorm_plans_of_the_bench_workloads(fk):
    # 16384 x 4096 fp32 and 65536 x 4096 bf16: 128 threads, 32 values each
    assert fk.fk_layernorm_rows_plan(16384, 4096, 0).as_dict()["threads"] == 128
    assert fk.fk_layernorm_rows_plan(65536, 4096, 1).as_dict()["vpt"] * 8 == 32


def test_layernorm_forced_plans_and_errors(fk):
    P = fk
    assert P.fk_layernorm_rows_plan(2, 100, 0, P.FK_PATH_CTA).as_dict()["path"] == "cta"
    assert P.fk_layernorm_rows_plan(2, 100, 0, P.FK_PATH_TWOPHASE).as_dict()["threads"] == 512
    with pytest.raises(P.FkError):
        P.fk_layernorm_rows_plan(2, 32769, 0, P.FK_PATH_CTA)     # more than a block holds
    with pytest.raises(P.FkError):
        P.fk_layernorm_rows_plan(2, 1025, 0, P.FK_PATH_WARP)     # more than a warp holds
    with pytest.raises(P.FkError):
        P.fk_layernorm_rows_plan(2, 4096, 0, P.FK_PATH_CLUSTER)  # no cluster path for LayerNorm
    with pytest.raises(P.FkError) as e:
        P.fk_layernorm_rows_plan(2, 10, 7)
    assert e.value.status == P.FK_ERR_UNSUPPORTED_DTYPE
    with pytest.raises(P.FkError):
        P.fk_layernorm_rows_plan(2, 0, 0)
