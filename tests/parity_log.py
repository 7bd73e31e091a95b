"""Errors of every parity comparison made in this pytest session, printed in
the terminal summary (also under -q) so that the margin to each tolerance is
on record, not only pass / fail."""
RECORDS = []


def record(what: str, max_abs: float, rel_l2: float, tol: dict, dtype: str):
    RECORDS.append((what, dtype, max_abs, rel_l2, tol["max_abs"], tol["rel_l2"]))
