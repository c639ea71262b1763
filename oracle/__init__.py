"""CPU oracle for the StagQ GEMV (test infrastructure; see stagq.py)."""
