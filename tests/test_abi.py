"""The C ABI library loads and exports every function include/slim.h declares.

No compute call is made here: only host-side queries and argument checks that
return before any device work.
"""
import ctypes

import pytest

from post_weight_quantization_hessian_b200 import build, slim


@pytest.fixture(scope="module")
def lib():
    build.build()
    return slim._lib()


def test_every_header_function_is_exported(lib):
    names = slim.header_functions()
    assert len(names) >= 17
    cdll = ctypes.CDLL(slim.LIB_PATH)
    missing = [n for n in names if not hasattr(cdll, n)]
    assert not missing, missing
    assert set(names) == set(slim._SIGS), "binding and header disagree"


def test_host_queries(lib):
    assert slim.slim_num_candidates(4096, 128) == 17          # k = 32 -> p in [0, 16]
    assert slim.slim_num_candidates(11008, 128) == 44
    assert slim.slim_num_candidates(5120, 32) == 81
    assert slim.slim_num_candidates(100, 32) == -1
    assert slim.slim_row_words(4096, 2) == 256
    assert lib.slim_status_string(5).decode() == "damped Hessian is not positive definite"
    assert lib.slim_status_string(99).decode() == "unknown status"
    assert "sm_100a" in slim.slim_version()
    ws = slim.slim_workspace_bytes(4096, 4096, 262144, 1, 128, 2)
    assert ws > 4096 * 4096 * 8                                # holds at least H in fp64
    assert slim.slim_workspace_bytes(4096, 4000, 262144, 1, 128, 2) == 0   # n % group != 0


@pytest.mark.parametrize("kw, why", [
    (dict(group=96), "group not in {32, 64, 128}"),
    (dict(n=640 + 32), "n % group != 0"),
    (dict(avg_bits=1), "avg_bits - 1 would be 0"),
    (dict(avg_bits=8), "avg_bits + 1 would exceed 8"),
    (dict(lam=1.0), "lambda >= 1"),
    (dict(lam=-0.1), "lambda < 0"),
    (dict(n_tau=0), "no tau candidate"),
    (dict(n_tau=300), "tau index must fit a byte"),
    (dict(N=0), "no tokens"),
    (dict(xdtype=5), "unknown X dtype"),
    (dict(W=0), "NULL weight"),
    (dict(W=0x1004), "W not 16-byte aligned"),
])
def test_layer_argument_validation(lib, kw, why):
    a = dict(W=0x1000, m=256, n=640, X=0x2000, xdtype=1, N=1000, group=128, avg_bits=2, lam=0.1, n_tau=50)
    a.update(kw)
    rc = lib.slim_quantize_layer(a["W"], a["m"], a["n"], a["X"], a["xdtype"], a["N"], a["group"], a["avg_bits"],
                                 a["lam"], a["n_tau"], 0x3000, 0x4000, 0x5000, 0x6000, None, 0, None)
    assert rc == 1, why


def test_stage_argument_validation(lib):
    assert lib.slim_hessian(0x1000, 1, 100, 48, 0x2000, None, 0, None) == 1        # n % 32 != 0
    assert lib.slim_hinv_diag(0x1000, 64, -1.0, 0x2000, None, 0, None) == 1      # negative damping
    assert lib.slim_salience(0x1000, 8, 256, 0x2000, 64, None, 0x3000, None, 0, None) == 1  # NULL S
    assert lib.slim_sqc(0x1000, 8, 256, 0x2000, 0x3000, 128, 2, 0.1, 0, 1, 2, 3, None, None) == 1


@pytest.mark.parametrize("m, n, N, xdtype, group", [
    (4096, 4096, 262144, 1, 128), (4096, 11008, 262144, 1, 128), (13824, 5120, 262144, 1, 32),
    (256, 512, 2048, 0, 128), (300, 640, 5000, 1, 64)])
def test_workspace_sizes(lib, m, n, N, xdtype, group):
    """Workspace sizes are pure host arithmetic: the split search needs the one-pass
    search's workspace plus its stored phase-A state (8 bytes per token tile row and
    output column, tiles padded to 128), and the whole layer holds H and the SBA
    operands at least."""
    one = lib.slim_sba_workspace_bytes(m, n, N, xdtype, group)
    split = lib.slim_sba_split_workspace_bytes(m, n, N, xdtype, group)
    tiles_t, tiles_o = -(-N // 128), -(-m // 128)
    assert split >= one + tiles_t * tiles_o * 128 * 128 * 8
    assert split - one <= tiles_t * tiles_o * 128 * 128 * 8 + 512
    ksplit = 1 if xdtype == 1 else 2
    operands = 4 * m * n * 2 + N * n * 2 * ksplit                   # three RTN arrays, W, X as fp16
    assert one >= operands
    layer = lib.slim_workspace_bytes(m, n, N, xdtype, group, 2)
    assert layer >= n * n * 8 + operands


def test_split_search_rejects_bad_chunks_before_any_launch(lib):
    for chunk in (0, -256, 100, 384):
        rc = lib.slim_sba_search_split(0x1000, 256, 512, 0x2000, 1, 4096, 128, 2, 0x3000, None, None, 0x4000, chunk,
                                       None, 0, None)
        assert rc == 1, chunk


def test_dequant_gemv_workspace_plan(lib):
    """The GEMV's shared-memory plan on the host: one launch (no workspace) when a
    block's 32 rows of words, scales, zeros and the batch's x fit; group ranges with
    fixed-order partials (workspace ks * batch * m floats) when they do not."""
    q = lib.slim_dequant_gemv_workspace_bytes
    assert q(13824, 5120, 32, 2, 1) == 0        # the 13B up_proj at group 32, batch 1
    assert q(4096, 4096, 128, 2, 1) == 0        # q_proj
    # down_proj (b 3): 32 rows of 1032 words each do not fit beside the rest: group ranges
    wd = q(4096, 11008, 128, 3, 1)
    assert wd > 0 and wd % (4096 * 4) == 0 and wd // (4096 * 4) >= 2
    w8 = q(13824, 5120, 32, 2, 8)               # batch 8: x of 8 rows no longer fits with the words
    assert w8 > 0 and w8 % (8 * 13824 * 4) == 0 and w8 // (8 * 13824 * 4) >= 2
    assert q(13824, 5120, 32, 2, 9) == 0        # batch above 8: not a valid call
    assert q(13824, 5100, 32, 2, 1) == 0        # n not a multiple of the group


def test_bench_traffic_record_follows_the_source():
    """bench.py reports the committed DRAM bytes of the scoring kernel only while the
    kernel's source is the one they were captured on."""
    import os
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    src = bench.source_hash("post_weight_quantization_hessian_b200/csrc/sba.cu",
                            "post_weight_quantization_hessian_b200/csrc/common.cuh")
    import json
    with open(os.path.join(root, "profiles", "traffic.json")) as f:
        stored = json.load(f)["sba_score_kernel"]["llama13b_up_proj_13824x5120_g32"]
    # the recorded bytes while the hash matches, nothing for any other source
    assert bench.traffic_record("sba_score_kernel", "llama13b_up_proj_13824x5120_g32",
                                stored["source_hash"]) == stored["bytes_per_launch"]
    rec = bench.traffic_record("sba_score_kernel", "llama13b_up_proj_13824x5120_g32", src)
    assert rec == (stored["bytes_per_launch"] if src == stored["source_hash"] else None)
    assert bench.traffic_record("sba_score_kernel", "llama13b_up_proj_13824x5120_g32", "0" * 16) is None
    assert bench.traffic_record("sba_score_kernel", "no_such_workload", src) is None
