"""Plant plausible page-gather mistakes in a copy of the oracle (CPU) and
check that at least one pin of tests/test_oracle_paged.py fails for each."""

import importlib

import numpy as np
import pytest

from tests.test_oracle_paged import PINS


def _fresh():
    spec = importlib.util.find_spec("oracle.diffattn")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _gather(m, order=1, extra=0, npg_floor=False, keep_all=False):
    """A gather_pages variant built from the module's own helpers."""
    def gather_pages(pages, table_row, n):
        pages = m._f64(pages)
        ps = pages.shape[1]
        npg = n // ps if npg_floor else -(-n // ps)
        row = np.asarray(table_row)
        if keep_all:
            npg = len(row)
        if npg == 0:
            return np.zeros((pages.shape[2], 0, pages.shape[3]))
        ids = row[:npg][::order]
        toks = np.concatenate([pages[int(p)] for p in ids], axis=0)
        toks = toks if keep_all else toks[:n + extra]
        return np.transpose(toks, (1, 0, 2))
    return gather_pages


def _mut_pages_reversed(m):
    m.gather_pages = _gather(m, order=-1)


def _mut_one_token_too_many(m):
    m.gather_pages = _gather(m, extra=1)


def _mut_one_token_too_few(m):
    m.gather_pages = _gather(m, extra=-1)


def _mut_page_count_floored(m):
    m.gather_pages = _gather(m, npg_floor=True)


def _mut_whole_table_read(m):
    m.gather_pages = _gather(m, keep_all=True)


def _mut_token_head_axes_swapped(m):
    """Token-major pages read as head-major: a reshape where a transpose belongs."""
    orig = m.gather_pages

    def gather_pages(pages, row, n):
        good = orig(pages, row, n)                        # [Hkv, n, D]
        toks = np.transpose(good, (1, 0, 2))              # back to the pages' [n, Hkv, D]
        return toks.reshape(good.shape)
    m.gather_pages = gather_pages


def _mut_first_sequence_table_for_all(m):
    orig = m.decode_v2_paged

    def decode_v2_paged(q, k_pages, v_pages, block_table, seq_lens, lam):
        bt = np.asarray(block_table.cpu() if hasattr(block_table, "cpu") else block_table).copy()
        bt[:] = bt[0]
        return orig(q, k_pages, v_pages, bt, seq_lens, lam)
    m.decode_v2_paged = decode_v2_paged


MUTATIONS = [_mut_pages_reversed, _mut_one_token_too_many, _mut_one_token_too_few, _mut_page_count_floored,
             _mut_whole_table_read, _mut_token_head_axes_swapped, _mut_first_sequence_table_for_all]


def _failures(m):
    failed = []
    for pin in PINS:
        try:
            pin(m)
        except Exception:
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("mutate", MUTATIONS, ids=lambda f: f.__name__)
def test_mutation_is_caught(mutate):
    m = _fresh()
    mutate(m)
    assert _failures(m), f"no pin catches {mutate.__name__}"


def test_unmutated_copy_passes():
    assert _failures(_fresh()) == []
