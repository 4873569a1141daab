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
