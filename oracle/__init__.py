"""fp64 CPU oracle for Ring Self-Attention: test infrastructure only (see ``oracle.py``)."""
