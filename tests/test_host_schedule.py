"""The product's budget schedule (host logic) agrees with the oracle's on
every step and block count of interest."""
from block_sparse_attention_36_b200 import schedule as prod
from oracle import schedule as ref


def test_budget_matches_oracle():
    for nb in (32, 256, 768, 929, 1000):
        for s in range(50):
            assert prod.keep_budget(s, nb) == ref.budget(s, nb)
            assert prod.is_refresh(s) == ref.is_refresh(s)
