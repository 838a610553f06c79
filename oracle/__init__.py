"""Float64 CPU oracle for HiLS attention (test infrastructure; see oracle.py)."""
